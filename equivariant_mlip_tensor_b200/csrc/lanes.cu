// Side streams ("lanes") of the library: launches of one call that write
// disjoint outputs run concurrently on lanes forked from the caller's stream
// with an event and joined back before the call returns, so the caller sees
// ordinary stream order.  One pool per (device, user) is created on first use
// and kept until the process exits.
#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <utility>

#include "launch.h"

namespace cgtp {

std::mutex& side_lanes_mutex(int pool) {
  static std::mutex mu[kLanePools];
  return mu[pool];
}

cudaError_t side_lanes(int pool, SideLanes** out) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, SideLanes> per_dev;
  if (pool < 0 || pool >= kLanePools) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = per_dev.find({dev, pool});
  if (it == per_dev.end()) {
    SideLanes L{};
    for (int k = 0; k < kMaxSideLanes && e == cudaSuccess; ++k) {
      e = cudaStreamCreateWithFlags(&L.side[k], cudaStreamNonBlocking);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L.join[k], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L.fork, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
    it = per_dev.emplace(std::make_pair(dev, pool), L).first;
  }
  *out = &it->second;
  return cudaSuccess;
}

cudaError_t lanes_fork(SideLanes* L, int n, cudaStream_t s) {
  if (n > kMaxSideLanes) return cudaErrorInvalidValue;
  cudaError_t e = cudaEventRecord(L->fork, s);
  for (int k = 0; k < n && e == cudaSuccess; ++k) e = cudaStreamWaitEvent(L->side[k], L->fork, 0);
  return e;
}

cudaError_t lanes_join(SideLanes* L, int n, cudaStream_t s) {
  cudaError_t err = cudaSuccess;
  for (int k = 0; k < n && k < kMaxSideLanes; ++k) {  // every lane, even after an error
    cudaError_t e = cudaEventRecord(L->join[k], L->side[k]);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, L->join[k], 0);
    if (err == cudaSuccess) err = e;
  }
  return err;
}

}  // namespace cgtp
