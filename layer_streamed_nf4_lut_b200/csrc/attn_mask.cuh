// Which keys a query sees, for the attention kernels (block-relative row indices).
//
// Plain layout (AttnShape.pl == 0): causal, key k visible to query q when k <= q.
// Shared-prefix pair layout (pl > 0): a block of S = pl + 2 rl rows holds [prefix | chosen
// response | rejected response]; segment 0 = prefix, 1 = chosen, 2 = rejected; a row's position
// is its index, minus rl for the rejected rows (the rejected response continues the prefix);
// a key is visible when it lies in the prefix or in the query's own segment, at a position not
// after the query's.
#pragma once
#include "internal.h"

namespace soup {

__host__ __device__ __forceinline__ int pk_seg(const AttnShape& s, int x) {
  return x < s.pl ? 0 : (x < s.pl + s.rl ? 1 : 2);
}
__host__ __device__ __forceinline__ int pk_pos(const AttnShape& s, int x) { return x < s.pl + s.rl ? x : x - s.rl; }
__host__ __device__ __forceinline__ bool visible(const AttnShape& s, int q, int k) {
  if (s.pl == 0) return k <= q;
  const int sk = pk_seg(s, k);
  return (sk == 0 || sk == pk_seg(s, q)) && pk_pos(s, k) <= pk_pos(s, q);
}

// True if some query row in [q0, q1) sees some key row in [k0, k1) (rows clipped to S).
__host__ __device__ __forceinline__ bool block_visible(const AttnShape& s, int q0, int q1, int k0, int k1) {
  q1 = q1 < s.S ? q1 : s.S;
  k1 = k1 < s.S ? k1 : s.S;
  if (q0 >= q1 || k0 >= k1) return false;
  if (s.pl == 0) return k0 <= q1 - 1;
  const int lo[3] = {0, s.pl, s.pl + s.rl}, hi[3] = {s.pl, s.pl + s.rl, s.S};
  for (int qs = 0; qs < 3; ++qs) {
    const int a0 = q0 > lo[qs] ? q0 : lo[qs], a1 = q1 < hi[qs] ? q1 : hi[qs];
    if (a0 >= a1) continue;
    for (int ks = 0; ks < 3; ++ks) {
      if (ks != 0 && ks != qs) continue;
      const int b0 = k0 > lo[ks] ? k0 : lo[ks], b1 = k1 < hi[ks] ? k1 : hi[ks];
      if (b0 >= b1) continue;
      if (pk_pos(s, b0) <= pk_pos(s, a1 - 1)) return true;
    }
  }
  return false;
}

}  // namespace soup
