// nm_select.cuh -- selection of the 2 survivors of a group of 4 bf16 weights
// (the 2:4 prune rule of "M:N sparsity on NVIDIA tensor cores": keep the two of
// largest magnitude; equal magnitudes go to the lower index; NaN above +Inf,
// NaNs tie).  Shared by the 2:4 compress kernels and the fused prune + GEMM.
// select_quad (two groups per call, 16-bit SIMD) is the fast form; select_pair
// takes one group.
#pragma once
#include <cstdint>

namespace nmk {

// Selection of one group.  Composite keys c_i = (magnitude field of e_i) * 4
// + (3 - i), NaNs folded to one key just above +Inf: all four are distinct,
// and a larger key means a larger magnitude or, on equal magnitudes, a lower
// index.  The two largest keys come from a four-input network (max/min of
// each pair, then the larger maximum and the larger of the smaller maximum and
// the larger minimum); their low bits give the positions.
__device__ __forceinline__ uint32_t ckey(uint32_t shifted_by2, uint32_t tie) {
  return min((shifted_by2 & 0x1FFFCu) | tie, 0x1FE04u | tie);  // 0x1FE04 = (0x7F81 << 2)
}

// Group of four in (lo, hi) = (e0 | e1 << 16, e2 | e3 << 16): returns the
// nibble p0 | p1 << 2 (p0 < p1), and in `pk` the two survivors (first in the
// low half).
__device__ __forceinline__ uint32_t select_pair(uint32_t lo, uint32_t hi, uint32_t& pk) {
  const uint32_t c0 = ckey(lo << 2, 3u), c1 = ckey(lo >> 14, 2u);
  const uint32_t c2 = ckey(hi << 2, 1u), c3 = ckey(hi >> 14, 0u);
  const uint32_t m01 = max(c0, c1), n01 = min(c0, c1);
  const uint32_t m23 = max(c2, c3), n23 = min(c2, c3);
  const uint32_t top = max(m01, m23);
  const uint32_t second = max(min(m01, m23), max(n01, n23));
  const uint32_t pa = (top & 3u) ^ 3u, pb = (second & 3u) ^ 3u;
  const uint32_t p0 = min(pa, pb), p1 = max(pa, pb);
  pk = __byte_perm(lo, hi, 0x1010u + p0 * 0x22u + p1 * 0x2200u);
  return p0 | (p1 << 2);
}

// Two groups at once, one in each 16-bit half of every register (16-bit SIMD):
// v = (x, y) group A, (z, w) group B, as in select_pair.  Returns the byte
// nibble_A | nibble_B << 4; pk_a / pk_b receive the two survivors of A / B.
// Element i of a group survives when it beats at least two of the other three,
// and i < j beats j exactly when |e_i| >= |e_j| (magnitude fields, NaN folded
// to one value just above +Inf).  Each comparison is the top bit of a 16-bit
// difference: with bit 15 set on the minuend, (0x8000 + m_i) - m_j keeps it
// exactly when m_i >= m_j, and no borrow crosses into the other half.
__device__ __forceinline__ uint32_t prmt_sign(uint32_t a, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(d) : "r"(a), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t select_quad(uint4 v, uint32_t& pk_a, uint32_t& pk_b) {
  const uint32_t X0 = __byte_perm(v.x, v.z, 0x5410u), X1 = __byte_perm(v.x, v.z, 0x7632u);
  const uint32_t X2 = __byte_perm(v.y, v.w, 0x5410u), X3 = __byte_perm(v.y, v.w, 0x7632u);
  const uint32_t M0 = __vminu2(X0 & 0x7FFF7FFFu, 0x7F817F81u), M1 = __vminu2(X1 & 0x7FFF7FFFu, 0x7F817F81u);
  const uint32_t M2 = __vminu2(X2 & 0x7FFF7FFFu, 0x7F817F81u), M3 = __vminu2(X3 & 0x7FFF7FFFu, 0x7F817F81u);
  const uint32_t S0 = M0 + 0x80008000u, S1 = M1 + 0x80008000u, S2 = M2 + 0x80008000u;
  const uint32_t c01 = S0 - M1, c02 = S0 - M2, c03 = S0 - M3, c12 = S1 - M2, c13 = S1 - M3, c23 = S2 - M3;
  // survivor flags in bits 15 and 31 (majority of the three comparisons)
  const uint32_t s0 = (c01 & c02) | (c01 & c03) | (c02 & c03);
  const uint32_t s1 = (~c01 & c12) | (~c01 & c13) | (c12 & c13);
  const uint32_t s2 = (~c02 & ~c12) | (~c02 & c23) | (~c12 & c23);
  const uint32_t s3 = (~c03 & ~c13) | (~c03 & ~c23) | (~c13 & ~c23);
  // flags to 16-bit masks: each byte takes the sign of byte 1 (low half) or byte 3 (high half)
  const uint32_t F0 = prmt_sign(s0, 0xBB99u), F1 = prmt_sign(s1, 0xBB99u);
  const uint32_t F2 = prmt_sign(s2, 0xBB99u), F3 = prmt_sign(s3, 0xBB99u);
  // first survivor: e0, else e1, else e2; second: e3, else e2, else e1
  const uint32_t first = (F0 & X0) | (~F0 & ((F1 & X1) | (~F1 & X2)));
  const uint32_t second = (F3 & X3) | (~F3 & ((F2 & X2) | (~F2 & X1)));
  pk_a = __byte_perm(first, second, 0x5410u);
  pk_b = __byte_perm(first, second, 0x7632u);
  // nibble p0 | p1 << 2 per group: A in bits 0..3, B in bits 20..23
  const uint32_t n = (~F0 & F1 & 0x00100001u) | (~F0 & ~F1 & 0x00200002u) | ((F3 | ~F2) & 0x00400004u) |
                     ((F3 | F2) & 0x00800008u);
  return (n | (n >> 16)) & 0xFFu;
}

}  // namespace nmk
