// Host-side Clebsch-Gordan table generator (see cg_table.cpp).
#pragma once

namespace cgtp {

// Dense real-basis block of path (l1, l2, l3) in [m1][m2][m3] order
// ((2l1+1)(2l2+1)(2l3+1) doubles).  *discarded (nullable) receives the
// largest magnitude of the part dropped by the real/imaginary choice.
// Zero block outside the triangle rule.
bool real_cg_block(int l1, int l2, int l3, double* out, double* discarded);

// Fills the packed constant tables: cg_table[kTableSize] in the layout of
// structure.h and shk[kShkSize] (harmonic normalisation constants).
// Returns 0, or a nonzero code if a self-check fails (1: a path is neither
// real nor imaginary, 2: a block is not unitary, 3: a coefficient falls
// outside the structural selection-rule pattern).
int build_constant_tables(float* cg_table, float* shk);

}  // namespace cgtp
