// Causal grouped-query attention, forward and backward, flash-style (sm_100a).
//
// q, k, v live in one [T, (hq + 2 hkv) d] bf16 buffer (the fused q|k|v projection output,
// RoPE already applied to q and k).  Query head h reads kv head h / (hq / hkv).
// Scores are scaled by 1/sqrt(d); the softmax runs online over 64-wide kv tiles with
// quad-shuffle row reductions; the forward saves the natural-log LSE per (b, h, s).
//
// Backward (no atomics, deterministic):
//   delta[t, h] = sum_d dO * O                                      (row kernel)
//   pass 1, one CTA per (kv tile, kv head): dV += P^T dO, dK += dS^T Q over every query head of
//           the group and every causal query tile, in a fixed order;
//   pass 2, one CTA per (query tile, head): dQ += dS K over the causal kv tiles.
//   P = exp(S - lse), dS = P * (dP - delta), dP = dO V^T.
//
// Shared-prefix pair blocks (AttnShape.pl > 0): [prefix | chosen | rejected] rows, the rejected
// response attending to the prefix and to itself only; a rejected query tile skips the chosen
// kv tiles, a chosen kv tile is read by chosen query tiles only.
//
// Tiles are 64 x 64; 4 warps each own 16 rows; bf16 m16n8k16 tensor-core MMAs with fp32
// accumulators, operands fed from padded shared memory by ldmatrix.
#include "common.cuh"
#include "internal.h"

namespace soup {

namespace {

constexpr int AT_BR = 64;
constexpr int AT_THREADS = 128;
constexpr float LOG2E = 1.4426950408889634f;

template <int D>
struct AttnCfg {
  static constexpr int LDS = D + 8;  // padded row (elements); 16-byte aligned, conflict-free ldmatrix
  static constexpr int TILE = AT_BR * LDS;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Visibility of key row k to query row q (block-relative).  Plain layout: causal.  Shared-
// prefix pair layout: segment 0 = prefix, 1 = chosen, 2 = rejected (rows pl + rl ..), position
// = row, minus rl for the rejected rows; a key is visible if it is in the prefix or in the
// query's own segment, at a position not after the query's.
__device__ __forceinline__ int pk_seg(const AttnShape& s, int x) { return x < s.pl ? 0 : (x < s.pl + s.rl ? 1 : 2); }
__device__ __forceinline__ int pk_pos(const AttnShape& s, int x) { return x < s.pl + s.rl ? x : x - s.rl; }
__device__ __forceinline__ bool visible(const AttnShape& s, int q, int k) {
  if (s.pl == 0) return k <= q;
  const int sk = pk_seg(s, k);
  return (sk == 0 || sk == pk_seg(s, q)) && pk_pos(s, k) <= pk_pos(s, q);
}
// kv tiles a query tile reads, in order: 0..qt, except that a rejected-response query tile
// skips the chosen response's tiles.  Returns the count; kv tile of step j = j + skip_at(j).
struct KvRange {
  int n, jump_from, jump;
};
__device__ __forceinline__ KvRange kv_range(const AttnShape& s, int qt) {
  KvRange r{qt + 1, 1 << 30, 0};
  if (s.pl > 0 && qt * AT_BR >= s.pl + s.rl) {
    r.jump_from = s.pl / AT_BR;
    r.jump = s.rl / AT_BR;
    r.n = qt + 1 - r.jump;
  }
  return r;
}
__device__ __forceinline__ int kv_tile(const KvRange& r, int j) { return j >= r.jump_from ? j + r.jump : j; }

// Load a 64 x D tile of rows [r0, r0+64) (rows >= nrows zero-filled) with cp.async.
template <int D>
__device__ __forceinline__ void load_tile_async(uint16_t* dst, const uint16_t* src, long long ld, int r0, int nrows) {
  constexpr int CH = D / 8;
  for (int c = threadIdx.x; c < AT_BR * CH; c += AT_THREADS) {
    const int r = c / CH, cc = c % CH;
    const bool ok = (r0 + r) < nrows;
    const uint16_t* g = src + static_cast<long long>(ok ? (r0 + r) : r0) * ld + cc * 8;
    cp_async16(dst + r * AttnCfg<D>::LDS + cc * 8, g, ok);
  }
}

// A fragment (16 rows x 16 cols at column k0) of a row-major padded tile, rows [row0, row0+16).
template <int D>
__device__ __forceinline__ void lda_frag(const uint16_t* tile, int row0, int k0, uint32_t (&a)[4]) {
  const int lane = threadIdx.x & 31;
  const int mi = lane >> 3, ri = lane & 7;
  const uint16_t* p = tile + (row0 + ri + (mi & 1) * 8) * AttnCfg<D>::LDS + k0 + (mi >> 1) * 8;
  ldsm_x4(smem_u32(p), a[0], a[1], a[2], a[3]);
}
// B fragments for two n8 blocks (rows n0..n0+15 of a [n][k] tile, k chunk k0..k0+15).
template <int D>
__device__ __forceinline__ void ldb_nk(const uint16_t* tile, int n0, int k0, uint32_t& b00, uint32_t& b01,
                                       uint32_t& b10, uint32_t& b11) {
  const int lane = threadIdx.x & 31;
  const int mi = lane >> 3, ri = lane & 7;
  const uint16_t* p = tile + (n0 + (mi >> 1) * 8 + ri) * AttnCfg<D>::LDS + k0 + (mi & 1) * 8;
  ldsm_x4(smem_u32(p), b00, b01, b10, b11);
}
// B fragments for two n8 blocks (columns n0..n0+15 of a [k][n] tile, k rows k0..k0+15).
template <int D>
__device__ __forceinline__ void ldb_kn(const uint16_t* tile, int k0, int n0, uint32_t& b00, uint32_t& b01,
                                       uint32_t& b10, uint32_t& b11) {
  const int lane = threadIdx.x & 31;
  const int mi = lane >> 3, ri = lane & 7;
  const uint16_t* p = tile + (k0 + (mi & 1) * 8 + ri) * AttnCfg<D>::LDS + n0 + (mi >> 1) * 8;
  ldsm_x4_t(smem_u32(p), b00, b01, b10, b11);
}

// ---------------------------------------------------------------- forward
template <int D>
__global__ void __launch_bounds__(AT_THREADS) attn_fwd_kernel(const AttnShape s, const uint16_t* __restrict__ qkv,
                                                               uint16_t* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(16) uint16_t sm[];
  using C = AttnCfg<D>;
  uint16_t* Qs = sm;
  uint16_t* Ks = sm + C::TILE;      // 2 buffers
  uint16_t* Vs = sm + 3 * C::TILE;  // 2 buffers
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (s.hq / s.hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row_base = static_cast<long long>(b) * s.S;
  const uint16_t* qsrc = qkv + row_base * s.ld_qkv + h * D;
  const uint16_t* ksrc = qkv + row_base * s.ld_qkv + (s.hq + g) * D;
  const uint16_t* vsrc = qkv + row_base * s.ld_qkv + (s.hq + s.hkv + g) * D;
  const float scale_log2 = LOG2E / sqrtf(static_cast<float>(D));

  const KvRange kr = kv_range(s, qt);
  const int nkv = kr.n;
  load_tile_async<D>(Qs, qsrc, s.ld_qkv, qt * AT_BR, s.S);
  load_tile_async<D>(Ks, ksrc, s.ld_qkv, kv_tile(kr, 0) * AT_BR, s.S);
  load_tile_async<D>(Vs, vsrc, s.ld_qkv, kv_tile(kr, 0) * AT_BR, s.S);
  cp_async_commit();

  float oacc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const int qrow0 = qt * AT_BR + warp * 16 + (lane >> 2);

  for (int j = 0; j < nkv; ++j) {
    if (j + 1 < nkv) {
      load_tile_async<D>(Ks + ((j + 1) & 1) * C::TILE, ksrc, s.ld_qkv, kv_tile(kr, j + 1) * AT_BR, s.S);
      load_tile_async<D>(Vs + ((j + 1) & 1) * C::TILE, vsrc, s.ld_qkv, kv_tile(kr, j + 1) * AT_BR, s.S);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint16_t* Kt = Ks + (j & 1) * C::TILE;
    const uint16_t* Vt = Vs + (j & 1) * C::TILE;
    const int kt = kv_tile(kr, j);
    float sacc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll
    for (int kc = 0; kc < D / 16; ++kc) {
      uint32_t a[4];
      lda_frag<D>(Qs, warp * 16, kc * 16, a);
#pragma unroll
      for (int nb2 = 0; nb2 < 4; ++nb2) {
        uint32_t b00, b01, b10, b11;
        ldb_nk<D>(Kt, nb2 * 16, kc * 16, b00, b01, b10, b11);
        mma16816(sacc[2 * nb2], a, b00, b01);
        mma16816(sacc[2 * nb2 + 1], a, b10, b11);
      }
    }
    // scale, causal mask, online softmax
    float mx[2] = {m_r[0], m_r[1]};
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kv = kt * AT_BR + nb * 8 + (lane & 3) * 2 + (e & 1);
        const int qi = qrow0 + (e >> 1) * 8;
        float v = sacc[nb][e] * scale_log2;
        if (!visible(s, qi, kv) || kv >= s.S) v = -INFINITY;
        sacc[nb][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    float corr[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      corr[r] = (mx[r] == -INFINITY) ? 1.f : exp2f(m_r[r] - mx[r]);
      m_r[r] = mx[r];
      l_r[r] *= corr[r];
    }
    uint32_t pa[4][4];  // P as A fragments, 4 k16 chunks over the 64 kv columns
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float mm = m_r[e >> 1];
        p[e] = (mm == -INFINITY) ? 0.f : exp2f(sacc[nb][e] - mm);
        l_r[e >> 1] += p[e];
      }
      pa[nb >> 1][(nb & 1) * 2 + 0] = pack_bf16x2(p[0], p[1]);
      pa[nb >> 1][(nb & 1) * 2 + 1] = pack_bf16x2(p[2], p[3]);
    }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      oacc[i][0] *= corr[0];
      oacc[i][1] *= corr[0];
      oacc[i][2] *= corr[1];
      oacc[i][3] *= corr[1];
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t a[4] = {pa[c][0], pa[c][1], pa[c][2], pa[c][3]};
#pragma unroll
      for (int db = 0; db < D / 8; db += 2) {
        uint32_t b00, b01, b10, b11;
        ldb_kn<D>(Vt, c * 16, db * 8, b00, b01, b10, b11);
        mma16816(oacc[db], a, b00, b01);
        mma16816(oacc[db + 1], a, b10, b11);
      }
    }
    __syncthreads();
  }
  // finalize
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qi = qrow0 + r * 8;
    if (qi >= s.S) continue;
    const float inv = 1.f / l_r[r];
    uint16_t* orow = out + (row_base + qi) * static_cast<long long>(s.hq * D) + h * D;
#pragma unroll
    for (int db = 0; db < D / 8; ++db) {
      const int col = db * 8 + (lane & 3) * 2;
      *reinterpret_cast<uint32_t*>(orow + col) = pack_bf16x2(oacc[db][2 * r] * inv, oacc[db][2 * r + 1] * inv);
    }
    if ((lane & 3) == 0)
      lse[(static_cast<long long>(b) * s.hq + h) * s.S + qi] = (m_r[r] + log2f(l_r[r])) / LOG2E;
  }
}

// ---------------------------------------------------------------- delta = rowsum(dO * O)
__global__ void attn_delta_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout, int T, int hq,
                                  int d, float* __restrict__ delta) {
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<long long>(T) * hq) return;
  const long long t = w / hq;
  const int h = static_cast<int>(w % hq);
  const uint16_t* a = o + t * hq * d + h * d;
  const uint16_t* b = dout + t * hq * d + h * d;
  float acc = 0.f;
  for (int c = lane * 2; c < d; c += 64) {
    const float2 x = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(a + c));
    const float2 y = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(b + c));
    acc += x.x * y.x + x.y * y.y;
  }
  acc = warp_sum(acc);
  if (lane == 0) delta[t * hq + h] = acc;  // [T, hq]
}

// ---------------------------------------------------------------- backward pass 1: dK, dV
// One CTA per (kv tile, kv head, head slice): it loops over the query heads of its slice of
// the group and over the causal query tiles, with the next (head, query tile) pair's Q / dO
// tiles loaded while the current one computes.  hsplit = 1: dK / dV go straight to dqkv.
// hsplit > 1 (too few kv tiles x kv heads to fill the GPU): each slice writes fp32 partial
// dK (scaled) / dV to part[slice][row][kv head][2D] and attn_dkdv_sum_kernel adds the slices
// in slice order.
template <int D>
__global__ void __launch_bounds__(AT_THREADS) attn_bwd_dkdv_kernel(const AttnShape s, const uint16_t* __restrict__ qkv,
                                                                    const uint16_t* __restrict__ dout,
                                                                    const float* __restrict__ lse,
                                                                    const float* __restrict__ delta,
                                                                    uint16_t* __restrict__ dqkv, int hsplit,
                                                                    float* __restrict__ part) {
  extern __shared__ __align__(16) uint16_t sm[];
  using C = AttnCfg<D>;
  uint16_t* Ks = sm;
  uint16_t* Vs = sm + C::TILE;
  uint16_t* Qb = sm + 2 * C::TILE;   // 2 buffers
  uint16_t* dOb = sm + 4 * C::TILE;  // 2 buffers
  float* lse_b = reinterpret_cast<float*>(sm + 6 * C::TILE);  // 2 x AT_BR
  float* del_b = lse_b + 2 * AT_BR;                            // 2 x AT_BR
  const int kt = blockIdx.x, b = blockIdx.z;
  const int g = blockIdx.y / hsplit, slice = blockIdx.y % hsplit;
  const int grp = s.hq / s.hkv;
  const int hper = grp / hsplit;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row_base = static_cast<long long>(b) * s.S;
  const long long ldo = static_cast<long long>(s.hq) * D;
  const float scale = 1.f / sqrtf(static_cast<float>(D));
  const float scale_log2 = scale * LOG2E;
  const int nqt = (s.S + AT_BR - 1) / AT_BR;
  // query tiles that see this kv tile: kt.. to the end, but a chosen-response kv tile of a
  // shared-prefix pair is seen by the chosen response only
  const int q_end = (s.pl > 0 && kt * AT_BR >= s.pl && kt * AT_BR < s.pl + s.rl) ? (s.pl + s.rl) / AT_BR : nqt;
  const int nq = q_end - kt;
  const int n_it = hper * nq;      // (head, query tile) pairs

  auto issue = [&](int it) {
    const int h = g * grp + slice * hper + it / nq;
    const int qt = kt + it % nq;
    const int buf = it & 1;
    load_tile_async<D>(Qb + buf * C::TILE, qkv + row_base * s.ld_qkv + h * D, s.ld_qkv, qt * AT_BR, s.S);
    load_tile_async<D>(dOb + buf * C::TILE, dout + row_base * ldo + h * D, ldo, qt * AT_BR, s.S);
    for (int i = threadIdx.x; i < AT_BR; i += AT_THREADS) {
      const int qi = qt * AT_BR + i;
      const bool ok = qi < s.S;
      lse_b[buf * AT_BR + i] = ok ? lse[(static_cast<long long>(b) * s.hq + h) * s.S + qi] * LOG2E : 0.f;
      del_b[buf * AT_BR + i] = ok ? delta[(row_base + qi) * s.hq + h] : 0.f;
    }
  };

  load_tile_async<D>(Ks, qkv + row_base * s.ld_qkv + (s.hq + g) * D, s.ld_qkv, kt * AT_BR, s.S);
  load_tile_async<D>(Vs, qkv + row_base * s.ld_qkv + (s.hq + s.hkv + g) * D, s.ld_qkv, kt * AT_BR, s.S);
  issue(0);
  cp_async_commit();

  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    dk[i][0] = dk[i][1] = dk[i][2] = dk[i][3] = 0.f;
    dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;
  }
  const int kvrow0 = kt * AT_BR + warp * 16 + (lane >> 2);

  for (int it = 0; it < n_it; ++it) {
    if (it + 1 < n_it) issue(it + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int qt = kt + it % nq;
    const uint16_t* Qs = Qb + (it & 1) * C::TILE;
    const uint16_t* dOs = dOb + (it & 1) * C::TILE;
    const float* lse_s = lse_b + (it & 1) * AT_BR;
    const float* del_s = del_b + (it & 1) * AT_BR;
    // S^T = K_w Q^T  (rows: kv, cols: q)
    float st[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) st[i][0] = st[i][1] = st[i][2] = st[i][3] = 0.f;
#pragma unroll
    for (int kc = 0; kc < D / 16; ++kc) {
      uint32_t a[4];
      lda_frag<D>(Ks, warp * 16, kc * 16, a);
#pragma unroll
      for (int nb2 = 0; nb2 < 4; ++nb2) {
        uint32_t b00, b01, b10, b11;
        ldb_nk<D>(Qs, nb2 * 16, kc * 16, b00, b01, b10, b11);
        mma16816(st[2 * nb2], a, b00, b01);
        mma16816(st[2 * nb2 + 1], a, b10, b11);
      }
    }
    // P^T
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qcol = nb * 8 + (lane & 3) * 2 + (e & 1);
        const int qi = qt * AT_BR + qcol;
        const int kv = kvrow0 + (e >> 1) * 8;
        float p = exp2f(st[nb][e] * scale_log2 - lse_s[qcol]);
        if (!visible(s, qi, kv) || qi >= s.S || kv >= s.S) p = 0.f;
        st[nb][e] = p;
      }
    }
    // dV += P^T dO
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t a[4] = {pack_bf16x2(st[2 * c][0], st[2 * c][1]), pack_bf16x2(st[2 * c][2], st[2 * c][3]),
                             pack_bf16x2(st[2 * c + 1][0], st[2 * c + 1][1]),
                             pack_bf16x2(st[2 * c + 1][2], st[2 * c + 1][3])};
#pragma unroll
      for (int db = 0; db < D / 8; db += 2) {
        uint32_t b00, b01, b10, b11;
        ldb_kn<D>(dOs, c * 16, db * 8, b00, b01, b10, b11);
        mma16816(dv[db], a, b00, b01);
        mma16816(dv[db + 1], a, b10, b11);
      }
    }
    // dP^T = V_w dO^T
    float dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
#pragma unroll
    for (int kc = 0; kc < D / 16; ++kc) {
      uint32_t a[4];
      lda_frag<D>(Vs, warp * 16, kc * 16, a);
#pragma unroll
      for (int nb2 = 0; nb2 < 4; ++nb2) {
        uint32_t b00, b01, b10, b11;
        ldb_nk<D>(dOs, nb2 * 16, kc * 16, b00, b01, b10, b11);
        mma16816(dp[2 * nb2], a, b00, b01);
        mma16816(dp[2 * nb2 + 1], a, b10, b11);
      }
    }
    // dS^T = P^T * (dP^T - delta), then dK += dS^T Q
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qcol = nb * 8 + (lane & 3) * 2 + (e & 1);
        st[nb][e] = st[nb][e] * (dp[nb][e] - del_s[qcol]);
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t a[4] = {pack_bf16x2(st[2 * c][0], st[2 * c][1]), pack_bf16x2(st[2 * c][2], st[2 * c][3]),
                             pack_bf16x2(st[2 * c + 1][0], st[2 * c + 1][1]),
                             pack_bf16x2(st[2 * c + 1][2], st[2 * c + 1][3])};
#pragma unroll
      for (int db = 0; db < D / 8; db += 2) {
        uint32_t b00, b01, b10, b11;
        ldb_kn<D>(Qs, c * 16, db * 8, b00, b01, b10, b11);
        mma16816(dk[db], a, b00, b01);
        mma16816(dk[db + 1], a, b10, b11);
      }
    }
    __syncthreads();  // this buffer is refilled two iterations later
  }
  // store dK (scaled) and dV: into the k / v columns of dqkv, or as fp32 partials
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int kv = kvrow0 + r * 8;
    if (kv >= s.S) continue;
    if (hsplit == 1) {
      uint16_t* krow = dqkv + (row_base + kv) * s.ld_qkv + (s.hq + g) * D;
      uint16_t* vrow = dqkv + (row_base + kv) * s.ld_qkv + (s.hq + s.hkv + g) * D;
#pragma unroll
      for (int db = 0; db < D / 8; ++db) {
        const int col = db * 8 + (lane & 3) * 2;
        *reinterpret_cast<uint32_t*>(krow + col) = pack_bf16x2(dk[db][2 * r] * scale, dk[db][2 * r + 1] * scale);
        *reinterpret_cast<uint32_t*>(vrow + col) = pack_bf16x2(dv[db][2 * r], dv[db][2 * r + 1]);
      }
    } else {
      const long long T = static_cast<long long>(s.B) * s.S;
      float* prow = part + ((static_cast<long long>(slice) * T + row_base + kv) * s.hkv + g) * (2 * D);
#pragma unroll
      for (int db = 0; db < D / 8; ++db) {
        const int col = db * 8 + (lane & 3) * 2;
        *reinterpret_cast<float2*>(prow + col) = make_float2(dk[db][2 * r] * scale, dk[db][2 * r + 1] * scale);
        *reinterpret_cast<float2*>(prow + D + col) = make_float2(dv[db][2 * r], dv[db][2 * r + 1]);
      }
    }
  }
}

// Sum of the head-slice partials in slice order -> bf16 dK / dV columns of dqkv.  One thread
// per 4 consecutive values of one row's [hkv][2D] block.
__global__ void attn_dkdv_sum_kernel(const AttnShape s, int hsplit, const float* __restrict__ part,
                                     uint16_t* __restrict__ dqkv) {
  const long long T = static_cast<long long>(s.B) * s.S;
  const int per_row = s.hkv * 2 * s.d;
  const long long idx = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (idx >= T * per_row) return;
  const long long row = idx / per_row;
  const int c = static_cast<int>(idx % per_row);
  const int g = c / (2 * s.d), w = c % (2 * s.d);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int sl = 0; sl < hsplit; ++sl) {
    const float4 v = *reinterpret_cast<const float4*>(part + (static_cast<long long>(sl) * T + row) * per_row + c);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  const int col = (w < s.d) ? (s.hq + g) * s.d + w : (s.hq + s.hkv + g) * s.d + (w - s.d);
  uint2* o = reinterpret_cast<uint2*>(dqkv + row * s.ld_qkv + col);
  *o = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
}

// ---------------------------------------------------------------- backward pass 2: dQ
template <int D>
__global__ void __launch_bounds__(AT_THREADS) attn_bwd_dq_kernel(const AttnShape s, const uint16_t* __restrict__ qkv,
                                                                  const uint16_t* __restrict__ dout,
                                                                  const float* __restrict__ lse,
                                                                  const float* __restrict__ delta,
                                                                  uint16_t* __restrict__ dqkv) {
  extern __shared__ __align__(16) uint16_t sm[];
  using C = AttnCfg<D>;
  uint16_t* Qs = sm;
  uint16_t* dOs = sm + C::TILE;
  uint16_t* Ks = sm + 2 * C::TILE;  // 2 buffers
  uint16_t* Vs = sm + 4 * C::TILE;  // 2 buffers
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (s.hq / s.hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row_base = static_cast<long long>(b) * s.S;
  const long long ldo = static_cast<long long>(s.hq) * D;
  const float scale = 1.f / sqrtf(static_cast<float>(D));
  const float scale_log2 = scale * LOG2E;
  const uint16_t* ksrc = qkv + row_base * s.ld_qkv + (s.hq + g) * D;
  const uint16_t* vsrc = qkv + row_base * s.ld_qkv + (s.hq + s.hkv + g) * D;

  const KvRange kr = kv_range(s, qt);
  load_tile_async<D>(Qs, qkv + row_base * s.ld_qkv + h * D, s.ld_qkv, qt * AT_BR, s.S);
  load_tile_async<D>(dOs, dout + row_base * ldo + h * D, ldo, qt * AT_BR, s.S);
  load_tile_async<D>(Ks, ksrc, s.ld_qkv, kv_tile(kr, 0) * AT_BR, s.S);
  load_tile_async<D>(Vs, vsrc, s.ld_qkv, kv_tile(kr, 0) * AT_BR, s.S);
  cp_async_commit();

  const int qrow0 = qt * AT_BR + warp * 16 + (lane >> 2);
  float lse_r[2], del_r[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qi = qrow0 + r * 8;
    const bool ok = qi < s.S;
    lse_r[r] = ok ? lse[(static_cast<long long>(b) * s.hq + h) * s.S + qi] * LOG2E : 0.f;
    del_r[r] = ok ? delta[(row_base + qi) * s.hq + h] : 0.f;
  }
  float dq[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
  const int nkv = kr.n;
  for (int j = 0; j < nkv; ++j) {
    if (j + 1 < nkv) {
      load_tile_async<D>(Ks + ((j + 1) & 1) * C::TILE, ksrc, s.ld_qkv, kv_tile(kr, j + 1) * AT_BR, s.S);
      load_tile_async<D>(Vs + ((j + 1) & 1) * C::TILE, vsrc, s.ld_qkv, kv_tile(kr, j + 1) * AT_BR, s.S);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint16_t* Kt = Ks + (j & 1) * C::TILE;
    const uint16_t* Vt = Vs + (j & 1) * C::TILE;
    const int kt = kv_tile(kr, j);
    float sc[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
      dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
    }
#pragma unroll
    for (int kc = 0; kc < D / 16; ++kc) {
      uint32_t a[4], ad[4];
      lda_frag<D>(Qs, warp * 16, kc * 16, a);
      lda_frag<D>(dOs, warp * 16, kc * 16, ad);
#pragma unroll
      for (int nb2 = 0; nb2 < 4; ++nb2) {
        uint32_t b00, b01, b10, b11;
        ldb_nk<D>(Kt, nb2 * 16, kc * 16, b00, b01, b10, b11);
        mma16816(sc[2 * nb2], a, b00, b01);
        mma16816(sc[2 * nb2 + 1], a, b10, b11);
        ldb_nk<D>(Vt, nb2 * 16, kc * 16, b00, b01, b10, b11);
        mma16816(dp[2 * nb2], ad, b00, b01);
        mma16816(dp[2 * nb2 + 1], ad, b10, b11);
      }
    }
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kv = kt * AT_BR + nb * 8 + (lane & 3) * 2 + (e & 1);
        const int qi = qrow0 + (e >> 1) * 8;
        float p = exp2f(sc[nb][e] * scale_log2 - lse_r[e >> 1]);
        if (!visible(s, qi, kv) || kv >= s.S || qi >= s.S) p = 0.f;
        sc[nb][e] = p * (dp[nb][e] - del_r[e >> 1]);
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t a[4] = {pack_bf16x2(sc[2 * c][0], sc[2 * c][1]), pack_bf16x2(sc[2 * c][2], sc[2 * c][3]),
                             pack_bf16x2(sc[2 * c + 1][0], sc[2 * c + 1][1]),
                             pack_bf16x2(sc[2 * c + 1][2], sc[2 * c + 1][3])};
#pragma unroll
      for (int db = 0; db < D / 8; db += 2) {
        uint32_t b00, b01, b10, b11;
        ldb_kn<D>(Kt, c * 16, db * 8, b00, b01, b10, b11);
        mma16816(dq[db], a, b00, b01);
        mma16816(dq[db + 1], a, b10, b11);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qi = qrow0 + r * 8;
    if (qi >= s.S) continue;
    uint16_t* qrow = dqkv + (row_base + qi) * s.ld_qkv + h * D;
#pragma unroll
    for (int db = 0; db < D / 8; ++db) {
      const int col = db * 8 + (lane & 3) * 2;
      *reinterpret_cast<uint32_t*>(qrow + col) = pack_bf16x2(dq[db][2 * r] * scale, dq[db][2 * r + 1] * scale);
    }
  }
}

template <int D>
cudaError_t fwd_d(const AttnShape& s, const uint16_t* qkv, uint16_t* o, float* lse, cudaStream_t st) {
  const int smem = 5 * AttnCfg<D>::TILE * 2;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid((s.S + AT_BR - 1) / AT_BR, s.hq, s.B);
  attn_fwd_kernel<D><<<grid, AT_THREADS, smem, st>>>(s, qkv, o, lse);
  ++g_kernel_launches;
  return cudaGetLastError();
}

template <int D>
cudaError_t bwd_d(const AttnShape& s, const uint16_t* qkv, const uint16_t* o, const uint16_t* dout, const float* lse,
                  float* delta, uint16_t* dqkv, float* ws, size_t ws_bytes, cudaStream_t st) {
  const int smem1 = 6 * AttnCfg<D>::TILE * 2 + 4 * AT_BR * 4;
  const int smem2 = 6 * AttnCfg<D>::TILE * 2;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int T = s.B * s.S;
  const long long warps = static_cast<long long>(T) * s.hq;
  attn_delta_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, st>>>(o, dout, T, s.hq, D, delta);
  // head slices: the largest divisor of the group size that keeps the grid within two CTAs
  // per SM and whose partials fit the workspace
  const int nkt = (s.S + AT_BR - 1) / AT_BR;
  const long long base = static_cast<long long>(nkt) * s.hkv * s.B;
  const int grp = s.hq / s.hkv;
  const size_t per_slice = static_cast<size_t>(T) * s.hkv * 2 * D * sizeof(float);
  int hsplit = 1;
  for (int c = grp; c > 1; --c)
    if (grp % c == 0 && base * c <= 2 * 148 && ws && static_cast<size_t>(c) * per_slice <= ws_bytes) {
      hsplit = c;
      break;
    }
  dim3 g1(nkt, s.hkv * hsplit, s.B);
  attn_bwd_dkdv_kernel<D><<<g1, AT_THREADS, smem1, st>>>(s, qkv, dout, lse, delta, dqkv, hsplit, ws);
  g_kernel_launches += 2;
  if (hsplit > 1) {
    const long long n4 = static_cast<long long>(T) * s.hkv * 2 * D / 4;
    attn_dkdv_sum_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, st>>>(s, hsplit, ws, dqkv);
    ++g_kernel_launches;
  }
  dim3 g2(nkt, s.hq, s.B);
  attn_bwd_dq_kernel<D><<<g2, AT_THREADS, smem2, st>>>(s, qkv, dout, lse, delta, dqkv);
  ++g_kernel_launches;
  return cudaGetLastError();
}

}  // namespace

cudaError_t attn_fwd_launch(const AttnShape& s, const uint16_t* qkv, uint16_t* o, float* lse, cudaStream_t st) {
  if (s.B <= 0 || s.S <= 0) return cudaSuccess;
  if (s.hkv <= 0 || s.hq % s.hkv != 0 || s.ld_qkv % 8 != 0) return cudaErrorInvalidValue;
  if (s.pl < 0 || (s.pl > 0 && (s.pl % AT_BR || s.rl <= 0 || s.rl % AT_BR || s.S != s.pl + 2 * s.rl)))
    return cudaErrorInvalidValue;
  if (s.d == 128) return fwd_d<128>(s, qkv, o, lse, st);
  if (s.d == 64) return fwd_d<64>(s, qkv, o, lse, st);
  return cudaErrorInvalidValue;
}

cudaError_t attn_bwd_launch(const AttnShape& s, const uint16_t* qkv, const uint16_t* o, const uint16_t* dout,
                            const float* lse, float* delta, uint16_t* dqkv, float* ws, size_t ws_bytes,
                            cudaStream_t st) {
  if (s.B <= 0 || s.S <= 0) return cudaSuccess;
  if (s.hkv <= 0 || s.hq % s.hkv != 0 || s.ld_qkv % 8 != 0) return cudaErrorInvalidValue;
  if (s.pl < 0 || (s.pl > 0 && (s.pl % AT_BR || s.rl <= 0 || s.rl % AT_BR || s.S != s.pl + 2 * s.rl)))
    return cudaErrorInvalidValue;
  if (s.d == 128) return bwd_d<128>(s, qkv, o, dout, lse, delta, dqkv, ws, ws_bytes, st);
  if (s.d == 64) return bwd_d<64>(s, qkv, o, dout, lse, delta, dqkv, ws, ws_bytes, st);
  return cudaErrorInvalidValue;
}

}  // namespace soup
