"""Pins for the oracle's neighbour list (CPU only)."""
import numpy as np
import pytest

from equivariant_mlip_tensor_b200 import synthetic
from oracle import graph


def _pairs(nl):
    dst = graph.edge_dst(nl["row_ptr"])
    return dst, nl["col"]


@pytest.mark.parametrize("case", ["tiny", "bulk_small", "molecules_small"])
def test_row_loop_matches_dense_all_pairs(case):
    if case == "tiny":
        w = synthetic.tiny()
        args = (w.pos, w.rc, None, None)
    elif case == "bulk_small":
        w = synthetic.bulk(n=300)
        args = (w.pos, w.rc, w.box, None)
    else:
        w = synthetic.molecules(n_graphs=6)
        args = (w.pos, w.rc, None, w.graph_id)
    nl = graph.neighbour_list(*args)
    i, j, d = graph.neighbour_list_all_pairs_matrix(*args)
    dst, src = _pairs(nl)
    assert np.array_equal(dst, i) and np.array_equal(src, j)
    assert np.array_equal(nl["edge_vec"].view(np.uint32), d.view(np.uint32))


def test_symmetry_and_antisymmetric_vectors():
    w = synthetic.bulk(n=300)
    nl = graph.neighbour_list(w.pos, w.rc, w.box)
    dst, src = _pairs(nl)
    fwd = {(int(a), int(b)): k for k, (a, b) in enumerate(zip(dst, src))}
    for (a, b), k in fwd.items():
        r = fwd[(b, a)]
        assert np.array_equal(nl["edge_vec"][k], -nl["edge_vec"][r])


def test_strict_cutoff_and_self_exclusion():
    pos = np.array([[0, 0, 0], [3, 0, 0], [0, 2.5, 0], [0, 2.5, 0]], dtype=np.float32)
    nl = graph.neighbour_list(pos, 3.0)
    dst, src = _pairs(nl)
    pairs = set(zip(dst.tolist(), src.tolist()))
    assert (0, 1) not in pairs  # exactly at the cutoff: excluded (strict <)
    assert (0, 2) in pairs and (2, 3) in pairs  # coincident atoms are neighbours
    assert all(a != b for a, b in pairs)
    k = [n for n, p in enumerate(zip(dst, src)) if p == (2, 3)][0]
    assert np.all(nl["edge_vec"][k] == 0.0)


def test_minimum_image():
    L = 10.0
    pos = np.array([[0.5, 5, 5], [9.6, 5, 5], [5, 5, 5]], dtype=np.float32)
    nl = graph.neighbour_list(pos, 2.0, box=L)
    dst, src = _pairs(nl)
    k = [n for n, p in enumerate(zip(dst, src)) if p == (0, 1)][0]
    want = np.float64(np.float32(9.6)) - np.float64(np.float32(0.5)) - 10.0
    assert nl["edge_vec"][k][0] == np.float32(want)
    assert len(dst) == 2
    with pytest.raises(ValueError):
        graph.neighbour_list(pos, 5.0, box=L)


def test_rint_ties_to_even():
    # d / L = 0.5 exactly: rint(0.5) = 0 keeps d; d / L = -0.5 also keeps d
    L = 4.0
    pos = np.array([[0, 0, 0], [2, 0, 0]], dtype=np.float32)
    d = graph.pair_displacements(pos, L)
    assert d[0, 1, 0] == 2.0 and d[1, 0, 0] == -2.0


def test_graph_ids_and_csc():
    w = synthetic.molecules(n_graphs=4)
    nl = graph.neighbour_list(w.pos, w.rc, None, w.graph_id)
    dst, src = _pairs(nl)
    assert np.all(w.graph_id[dst] == w.graph_id[src])
    # CSC lists, for each source, its edges in ascending destination
    ptr, ce, cd = nl["csc_ptr"], nl["csc_edge"], nl["csc_dst"]
    for j in range(w.n_nodes):
        es = ce[ptr[j]:ptr[j + 1]]
        assert np.all(src[es] == j)
        assert np.all(np.diff(dst[es]) > 0)
        assert np.array_equal(cd[ptr[j]:ptr[j + 1]], dst[es])
    assert np.array_equal(np.sort(ce), np.arange(src.size))
