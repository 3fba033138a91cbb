// nm_select.cuh -- selection of the 2 survivors of a group of 4 bf16 weights
// (the 2:4 prune rule of "M:N sparsity on NVIDIA tensor cores": keep the two of
// largest magnitude; equal magnitudes go to the lower index; NaN above +Inf,
// NaNs tie).  Shared by the 2:4 compress kernels.
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

}  // namespace nmk
