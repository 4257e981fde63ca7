// Causal grouped-query attention, forward and backward, on the tcgen05 tensor cores (sm_100a).
//
// One CTA per (128-query tile, query head, sequence).  q, k, v come from the fused
// [T, (hq + 2 hkv) d] bf16 projection output (RoPE applied) through TMA (128-byte swizzle); query
// head h reads kv head h / (hq / hkv).  Per 128-key tile j the CTA computes
//   S_j = Q K_j^T                      tcgen05.mma, both operands K-major in shared memory, fp32 in TMEM
//   P_j = exp(S_j / sqrt(d) - m)       softmax warps: one thread per query row reads its row of S_j
//                                      from TMEM, keeps the running max m and sum l, writes P_j back
//                                      to TMEM as bf16 over the first half of S_j's columns
//   O  = O * exp(m_old - m) + P_j V_j  the softmax warps rescale O in TMEM when m grows; P_j is the
//                                      MMA's A operand straight from TMEM, V_j the MN-major B operand
// and finally out = O / l, lse = m + log l (natural log) per row.  S/P use three TMEM buffers so
// that S_{j+1} is computed while the softmax of j runs and PV_{j-1} finishes; O takes d columns.
//
// Warp roles (192 threads): warps 0-3 softmax and epilogue (TMEM lane quarters 0-3, thread = query
// row), warp 4 allocates TMEM and its lane 0 issues the MMAs, warp 5 lane 0 issues the TMA loads
// (Q once; K and V tiles each in a 3-stage ring of its own, a K stage freed as soon as its S
// MMAs retire; one 3D copy per [128 rows x d] tile).  Every wait is bounded (mbar_wait_bounded):
// on timeout the device error word is set and the kernel runs to its end.
//
// Key tiles a query tile reads: those with a visible (query, key) pair (attn_mask.cuh); the plain
// causal layout reads tiles 0..qt.  Rows at or past S (a ragged last tile) are masked as keys and
// never stored as queries.
#include "attn_mask.cuh"
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"


namespace soup {

namespace {

constexpr int TQ = 128;  // query rows per CTA: one M = 128 accumulator
constexpr int TK = 128;  // keys per tile
constexpr int FWD_THREADS = 192;
constexpr int SOFTMAX_WARPS = 4;
constexpr int MMA_WARP = 4, TMA_WARP = 5;
constexpr int N_SBUF = 3;  // TMEM S/P buffers
constexpr float LOG2E_F = 1.4426950408889634f;

template <int D>
struct FwdCfg {
  static constexpr int TILE_BYTES = TQ * D * 2;  // one [128 x D] bf16 tile: D/64 swizzle atoms of 16 KB
  static constexpr int KV_STAGES = 3;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE_BYTES;                    // KV_STAGES stages
  static constexpr int V_OFF = (1 + KV_STAGES) * TILE_BYTES;  // KV_STAGES stages
  static constexpr int BAR_OFF = (1 + 2 * KV_STAGES) * TILE_BYTES;
  static constexpr int SMEM_BYTES = 1024 + BAR_OFF + 256;
  static_assert((1 + 4 * KV_STAGES + 2 * N_SBUF + 1 + 2) * 8 <= 256, "barrier block");
  static constexpr int O_COL = N_SBUF * TK;      // TMEM column of the O accumulator
  static constexpr int TMEM_COLS = 512;
  static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
};

// 2^x with the MUFU approximation (PTX ex2.approx.ftz: relative error about 2^-22), results below
// 2^-126 flushed to zero: a probability that small is zero at bf16 and in the fp32 row sum alike.
// The softmax rows' exponentials are the attention kernels' most frequent instruction.
__device__ __forceinline__ float exp2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Masks 32 consecutive scores of query row q (keys k0..k0+31) that the row must not see: keys
// at or past S and keys `visible` rejects become -inf.
__device__ __forceinline__ void mask_keys32(const AttnShape& s, int q, int k0, uint32_t (&raw)[32]) {
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const int k = k0 + e;
    if (k >= s.S || !visible(s, q, k)) raw[e] = 0xff800000u;  // -inf
  }
}

// Key tile j is read by query tile qt.
__device__ __forceinline__ bool kv_needed(const AttnShape& s, int qt, int j) {
  if (s.pl == 0) return j <= qt && j * TK < s.S;
  return block_visible(s, qt * TQ, qt * TQ + TQ, j * TK, j * TK + TK);
}

template <int D>
__global__ void __launch_bounds__(FWD_THREADS, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap tmap_o,
                       const AttnShape s, uint16_t* __restrict__ out, float* __restrict__ lse, int* err) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::BAR_OFF);
  // K and V stages have barriers of their own: K_j's stage frees when S_j's MMAs retire, long
  // before V_j's (after PV_j), so the next K tiles load while the softmax runs
  constexpr int KS = C::KV_STAGES;
  uint64_t* q_full = bars;                 // 1
  uint64_t* k_full = bars + 1;             // KS
  uint64_t* v_full = k_full + KS;          // KS
  uint64_t* k_empty = v_full + KS;         // KS
  uint64_t* v_empty = k_empty + KS;        // KS
  uint64_t* s_full = v_empty + KS;         // N_SBUF
  uint64_t* p_full = s_full + N_SBUF;      // N_SBUF
  uint64_t* o_ready = p_full + N_SBUF;     // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_ready + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(o_ready + 2);

  // the last query tiles see the most keys: they start first (longest work first on the SMs)
  const int qt = gridDim.x - 1 - blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (s.hq / s.hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntk = (s.S + TK - 1) / TK;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < N_SBUF; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], SOFTMAX_WARPS);
    }
    mbar_init(o_ready, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int row0 = b * s.S;  // first row of this sequence in the qkv buffer

  if (warp == TMA_WARP) {
    if (lane == 0) {
      constexpr uint32_t TB = C::TILE_BYTES;
      mbar_arrive_expect_tx(q_full, TB);
      tma_load_3d(base + C::Q_OFF, &tmap, 0, row0 + qt * TQ, h * (D / 64), q_full);
      int jj = 0;
      for (int j = 0; j < ntk; ++j) {
        if (!kv_needed(s, qt, j)) continue;
        const int st = jj % KS;
        const uint32_t ph = static_cast<uint32_t>((jj / KS) & 1) ^ 1u;
        mbar_wait_bounded(&k_empty[st], ph, abort_flag, err);
        mbar_arrive_expect_tx(&k_full[st], TB);
        tma_load_3d(base + C::K_OFF + st * TB, &tmap, 0, row0 + j * TK, (s.hq + g) * (D / 64), &k_full[st]);
        mbar_wait_bounded(&v_empty[st], ph, abort_flag, err);
        mbar_arrive_expect_tx(&v_full[st], TB);
        tma_load_3d(base + C::V_OFF + st * TB, &tmap, 0, row0 + j * TK, (s.hq + s.hkv + g) * (D / 64), &v_full[st]);
        ++jj;
      }
    }
  } else if (warp == MMA_WARP) {
    if (lane == 0) {
      const uint32_t sq = smem_u32(base + C::Q_OFF);
      const uint32_t idesc_qk = idesc_bf16(TQ, TK, false, false);  // S[q, k] = sum_d Q[q, d] K[k, d]
      const uint32_t idesc_pv = idesc_bf16(TQ, D, false, true);    // O[q, d] += sum_k P[q, k] V[k, d]
      mbar_wait_bounded(q_full, 0, abort_flag, err);
      auto issue_pv = [&](int i) {
        const int st = i % KS, sb = i % N_SBUF;
        mbar_wait_bounded(&v_full[st], (i / KS) & 1, abort_flag, err);
        mbar_wait_bounded(&p_full[sb], (i / N_SBUF) & 1, abort_flag, err);
        tc_fence_after();
        const uint32_t sv = smem_u32(base + C::V_OFF + st * C::TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < TK / 16; ++kk) {
          const uint64_t bd = sw128_mnmajor_desc(sv + kk * 2048, TK * 128);
          tc_mma_f16_ts(tmem + C::O_COL, tmem + sb * TK + kk * 8, bd, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&v_empty[st]);
        tc_commit(o_ready);
      };
      int jj = 0;
      for (int j = 0; j < ntk; ++j) {
        if (!kv_needed(s, qt, j)) continue;
        const int st = jj % KS, sb = jj % N_SBUF;
        mbar_wait_bounded(&k_full[st], (jj / KS) & 1, abort_flag, err);
        tc_fence_after();
        const uint32_t sk = smem_u32(base + C::K_OFF + st * C::TILE_BYTES);
#pragma unroll
        for (int kc = 0; kc < D / 16; ++kc) {
          const uint32_t off = (kc >> 2) * 16384 + (kc & 3) * 32;
          tc_mma_f16(tmem + sb * TK, sw128_kmajor_desc(sq + off), sw128_kmajor_desc(sk + off), idesc_qk,
                     kc > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[sb]);
        tc_commit(&k_empty[st]);  // K_jj's stage is free once S_jj's MMAs retire
        if (jj > 0) issue_pv(jj - 1);
        ++jj;
      }
      if (jj > 0) issue_pv(jj - 1);
    }
  } else {
    // ------------------------------------------------------ softmax: thread = query row
    const int r = warp * 32 + lane;
    const int q = qt * TQ + r;  // row within the sequence
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float scale_log2 = LOG2E_F / sqrtf(static_cast<float>(D));
    float m = -INFINITY, l = 0.f;
    int jj = 0;
    for (int j = 0; j < ntk; ++j) {
      if (!kv_needed(s, qt, j)) continue;
      const int sb = jj % N_SBUF;
      mbar_wait_bounded(&s_full[sb], (jj / N_SBUF) & 1, abort_flag, err);
      tc_fence_after();
      const bool need_mask = s.pl > 0 || j == qt || (j + 1) * TK > s.S;
      const uint32_t srow = tmem + lane_base + sb * TK;
      // the row's 128 scores come out of TMEM in four loads and one wait; then the tile's max,
      // and P = exp2(S scale - m) as bf16 over the first half of the buffer's columns (two per
      // column), the sum kept in four partial sums.  PV_{jj-1} reads another buffer, so this
      // may run before it has finished.
      uint32_t raw[TK / 32][32];
#pragma unroll
      for (int c = 0; c < TK / 32; ++c) tmem_ld32(srow + c * 32, raw[c]);
      tmem_ld_wait();
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < TK / 32; ++c) mask_keys32(s, q, j * TK + c * 32, raw[c]);
      }
      float t[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < TK / 32; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) t[e & 3] = fmaxf(t[e & 3], __uint_as_float(raw[c][e]));
      const float mx = fmaxf(m, fmaxf(fmaxf(t[0], t[1]), fmaxf(t[2], t[3])) * scale_log2);  // scale_log2 > 0
      const bool live = mx != -INFINITY;  // some key of this row visible so far
      const float alpha = live ? exp2f(m - mx) : 1.f;
      float sums[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < TK / 32; ++c) {
        uint32_t pw[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = live ? exp2_ftz(__uint_as_float(raw[c][e]) * scale_log2 - mx) : 0.f;
          const float p1 = live ? exp2_ftz(__uint_as_float(raw[c][e + 1]) * scale_log2 - mx) : 0.f;
          sums[e & 2] += p0;
          sums[(e & 2) + 1] += p1;
          pw[e >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st16(srow + c * 16, pw);
      }
      const float sum = (sums[0] + sums[1]) + (sums[2] + sums[3]);
      l = l * alpha + sum;
      m = mx;
      if (jj > 0) {
        // PV_{jj-1} has finished accumulating into O: rescale it where this row's max grew
        mbar_wait_bounded(o_ready, (jj - 1) & 1, abort_flag, err);
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 2
          for (int c = 0; c < D / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(tmem + lane_base + C::O_COL + c * 16, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st16(tmem + lane_base + C::O_COL + c * 16, o);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
      ++jj;
    }
    // epilogue: O / l in bf16, natural-log LSE.  A whole query tile is written into Q's shared
    // tile (free: every MMA has retired) in the TMA's swizzled layout and leaves in one TMA
    // store; a ragged last tile (its rows past S belong to the next sequence) stores row by row.
    if (jj > 0) mbar_wait_bounded(o_ready, (jj - 1) & 1, abort_flag, err);
    tc_fence_after();
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    const bool whole_tile = qt * TQ + TQ <= s.S;
    uint8_t* otile = base + C::Q_OFF;
    uint16_t* orow = out + (static_cast<long long>(row0) + q) * static_cast<long long>(s.hq * D) + h * D;
    // 64 columns of O per TMEM round trip (two loads, one wait), 16 per store step
#pragma unroll 1
    for (int c64 = 0; c64 < D / 64; ++c64) {
      uint32_t ov[2][32];
      tmem_ld32(tmem + lane_base + C::O_COL + c64 * 64, ov[0]);
      tmem_ld32(tmem + lane_base + C::O_COL + c64 * 64 + 32, ov[1]);
      tmem_ld_wait();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int c = c64 * 4 + cc;
        const uint32_t* o = &ov[cc >> 1][(cc & 1) * 16];
        uint4 w0, w1;
        w0.x = pack_bf16x2(__uint_as_float(o[0]) * inv, __uint_as_float(o[1]) * inv);
        w0.y = pack_bf16x2(__uint_as_float(o[2]) * inv, __uint_as_float(o[3]) * inv);
        w0.z = pack_bf16x2(__uint_as_float(o[4]) * inv, __uint_as_float(o[5]) * inv);
        w0.w = pack_bf16x2(__uint_as_float(o[6]) * inv, __uint_as_float(o[7]) * inv);
        w1.x = pack_bf16x2(__uint_as_float(o[8]) * inv, __uint_as_float(o[9]) * inv);
        w1.y = pack_bf16x2(__uint_as_float(o[10]) * inv, __uint_as_float(o[11]) * inv);
        w1.z = pack_bf16x2(__uint_as_float(o[12]) * inv, __uint_as_float(o[13]) * inv);
        w1.w = pack_bf16x2(__uint_as_float(o[14]) * inv, __uint_as_float(o[15]) * inv);
        if (whole_tile) {
          // columns 16c.. : plane 16c / 64, 16-byte chunks 2(c % 4) and 2(c % 4) + 1 of row r,
          // placed by the 128-byte swizzle (chunk index XOR row % 8)
          const uint32_t rowa = smem_u32(otile) + static_cast<uint32_t>((c >> 2) * (TQ * 128) + r * 128);
          const uint32_t ch = static_cast<uint32_t>((c & 3) * 2), sw = static_cast<uint32_t>(r & 7);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(rowa + ((ch ^ sw) << 4)), "r"(w0.x),
                       "r"(w0.y), "r"(w0.z), "r"(w0.w)
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(rowa + (((ch + 1) ^ sw) << 4)), "r"(w1.x),
                       "r"(w1.y), "r"(w1.z), "r"(w1.w)
                       : "memory");
        } else if (q < s.S) {
          *reinterpret_cast<uint4*>(orow + c * 16) = w0;
          *reinterpret_cast<uint4*>(orow + c * 16 + 8) = w1;
        }
      }
    }
    if (whole_tile) {
      fence_proxy_async_smem();  // the tile's generic-proxy writes, visible to the TMA
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (threadIdx.x == 0) {
        tma_store_3d(&tmap_o, 0, row0 + qt * TQ, h * (D / 64), otile);
        tma_store_commit_wait_read();
      }
    }
    if (q < s.S) lse[(static_cast<long long>(b) * s.hq + h) * s.S + q] = (m + log2f(l)) / LOG2E_F;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D>
cudaError_t launch_fwd(const AttnShape& s, const uint16_t* qkv, uint16_t* o, float* lse, int* err, cudaStream_t st) {
  using C = FwdCfg<D>;
  // one copy per [128 rows x D] tile: the head's D/64 column blocks as the planes of a 3D map
  CUtensorMap map, map_o;
  const unsigned long long planes = static_cast<unsigned long long>(s.hq + 2 * s.hkv) * (D / 64);
  const unsigned long long rows = static_cast<unsigned long long>(s.B) * s.S;
  if (!tma_encode_bf16_sw128_planes(&map, qkv, rows, planes, static_cast<unsigned long long>(s.ld_qkv) * 2, TQ, D / 64))
    return cudaErrorInvalidValue;
  // the output [T, hq d] as the same kind of map: a query tile's head is one [128 x D] box
  if (!tma_encode_bf16_sw128_planes(&map_o, o, rows, static_cast<unsigned long long>(s.hq) * (D / 64),
                                    static_cast<unsigned long long>(s.hq) * D * 2, TQ, D / 64))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    const cudaError_t e =
        cudaFuncSetAttribute(attn_fwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const dim3 grid((s.S + TQ - 1) / TQ, s.hq, s.B);
  attn_fwd_tc_kernel<D><<<grid, FWD_THREADS, C::SMEM_BYTES, st>>>(map, map_o, s, o, lse, err);
  return cudaGetLastError();
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

// ---------------------------------------------------------------- backward
// Two passes, no atomics (the result does not depend on timing), same arithmetic as the
// forward: P = exp(S / sqrt(d) - lse), dP = dO V^T, dS = P * (dP - delta), delta = rowsum(dO * O).
//   dK/dV pass, one CTA per (128-key tile, kv head, head slice); thread = key row:
//     S^T = K Q_i^T and dP^T = V dO_i^T (tcgen05, K-major operands), P^T and dS^T back into TMEM
//     as bf16 over the first half of their columns, then dV += P^T dO_i and dK += dS^T Q_i with
//     P^T / dS^T the A operands from TMEM and dO_i / Q_i read MN-major from the same shared tiles;
//     over the causal query tiles i of every query head of the slice.  One slice writes dK, dV
//     (bf16); several write fp32 partials that attn_dkdv_sum_kernel adds in slice order.
//   dQ pass, one CTA per (128-query tile, head); thread = query row:
//     S = Q K_j^T, dP = dO V_j^T, dS into TMEM, dQ += dS K_j (K_j read MN-major).
// The MMAs that overwrite S / dP wait until the previous iteration's MMAs reading P / dS from
// those columns have completed.
template <int D>
struct BwdCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int VEC_OFF = 6 * TILE_BYTES;  // two float[128] vectors (dK/dV pass)
  static constexpr int BAR_OFF = VEC_OFF + 1024;
  static constexpr int SMEM_BYTES = 1024 + BAR_OFF + 256;
  static constexpr int S_COL = 0, DP_COL = 128, ACC0 = 256, ACC1 = 256 + D;
  static constexpr int TMEM_COLS = 512;
  static_assert(ACC1 + D <= TMEM_COLS, "TMEM budget");
};

// K-major tile descriptors: 16-deep step kc of a [128 x D] tile (D/64 atoms of 16 KB)
__device__ __forceinline__ uint64_t kdesc(uint32_t tile, int kc) {
  return sw128_kmajor_desc(tile + (kc >> 2) * 16384 + (kc & 3) * 32);
}
// MN-major view of the same tile: rows are the reduction index, 16 rows per step
__device__ __forceinline__ uint64_t mndesc(uint32_t tile, int kk) { return sw128_mnmajor_desc(tile + kk * 2048, 128 * 128); }

// The RoPE backward on one row of dQ or dK: columns (i0.., i0 + d/2..) of a head rotated back by
// the angles of the row's position, x1' = x1 cos + x2 sin, x2' = x2 cos - x1 sin (no tables: no
// rotation).
template <int D>
__device__ __forceinline__ void rope_back16(const AttnShape& s, int pos, int i0, float (&x1)[16], float (&x2)[16]) {
  if (!s.rope_cos) return;
  const float4* cp = reinterpret_cast<const float4*>(s.rope_cos + static_cast<long long>(pos) * (D / 2) + i0);
  const float4* sp = reinterpret_cast<const float4*>(s.rope_sin + static_cast<long long>(pos) * (D / 2) + i0);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const float4 cv = __ldg(cp + g), sv = __ldg(sp + g);
    const float c[4] = {cv.x, cv.y, cv.z, cv.w}, sn[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float a = x1[4 * g + u], b = x2[4 * g + u];
      x1[4 * g + u] = a * c[u] + b * sn[u];
      x2[4 * g + u] = b * c[u] - a * sn[u];
    }
  }
}

__device__ __forceinline__ void store_bf16x16(uint16_t* dst, const float (&f)[16]) {
  reinterpret_cast<uint4*>(dst)[0] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                                pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
  reinterpret_cast<uint4*>(dst)[1] = make_uint4(pack_bf16x2(f[8], f[9]), pack_bf16x2(f[10], f[11]),
                                                pack_bf16x2(f[12], f[13]), pack_bf16x2(f[14], f[15]));
}
__device__ __forceinline__ void store_f32x16(float* dst, const float (&f)[16]) {
#pragma unroll
  for (int e = 0; e < 16; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
}

template <int D>
__global__ void __launch_bounds__(FWD_THREADS, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
                            const AttnShape s, const float* __restrict__ lse, const float* __restrict__ delta,
                            uint16_t* __restrict__ dqkv, int hsplit, float* __restrict__ part, int* err) {
  using C = BwdCfg<D>;
  constexpr int TB = C::TILE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* Ks = base;
  uint8_t* Vs = base + TB;
  uint8_t* Qs = base + 2 * TB;   // 2 stages
  uint8_t* dOs = base + 4 * TB;  // 2 stages
  float* lsm = reinterpret_cast<float*>(base + C::VEC_OFF);
  float* dsm = lsm + 128;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::BAR_OFF);
  uint64_t* kv_full = bars;       // 1
  uint64_t* qd_full = bars + 1;   // 2
  uint64_t* qd_empty = bars + 3;  // 2
  uint64_t* s_full = bars + 5;    // 1
  uint64_t* p_full = bars + 6;    // 1
  uint64_t* mma_done = bars + 7;  // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 9);

  const int j = blockIdx.x, b = blockIdx.z;
  const int g = blockIdx.y / hsplit, slice = blockIdx.y % hsplit;
  const int grp = s.hq / s.hkv, hper = grp / hsplit, h0 = g * grp + slice * hper;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqt = (s.S + TQ - 1) / TQ;
  const int row0 = b * s.S;
  const float scale = 1.f / sqrtf(static_cast<float>(D));
  const float scale_log2 = scale * LOG2E_F;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qd_full[i], 1);
      mbar_init(&qd_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, SOFTMAX_WARPS);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // iterations: (head hh of the slice, query tile i that sees key tile j), heads outer
  auto q_seen = [&](int i) { return block_visible(s, i * TQ, i * TQ + TQ, j * TK, j * TK + TK); };

  if (warp == TMA_WARP) {
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_full, 2 * TB);
      tma_load_3d(Ks, &tq, 0, row0 + j * TK, (s.hq + g) * (D / 64), kv_full);
      tma_load_3d(Vs, &tq, 0, row0 + j * TK, (s.hq + s.hkv + g) * (D / 64), kv_full);
      int it = 0;
      for (int hh = 0; hh < hper; ++hh)
        for (int i = 0; i < nqt; ++i) {
          if (!q_seen(i)) continue;
          const int h = h0 + hh, st = it & 1;
          mbar_wait_bounded(&qd_empty[st], ((it >> 1) & 1) ^ 1u, abort_flag, err);
          mbar_arrive_expect_tx(&qd_full[st], 2 * TB);
          tma_load_3d(Qs + st * TB, &tq, 0, row0 + i * TQ, h * (D / 64), &qd_full[st]);
          tma_load_3d(dOs + st * TB, &tdo, 0, row0 + i * TQ, h * (D / 64), &qd_full[st]);
          ++it;
        }
    }
  } else if (warp == MMA_WARP) {
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16(TK, TQ, false, false);  // [key, query], K = d
      const uint32_t idesc_a = idesc_bf16(TK, D, false, true);    // [key, d], K = queries
      const uint32_t sk = smem_u32(Ks), sv = smem_u32(Vs);
      mbar_wait_bounded(kv_full, 0, abort_flag, err);
      int it = 0;
      for (int hh = 0; hh < hper; ++hh)
        for (int i = 0; i < nqt; ++i) {
          if (!q_seen(i)) continue;
          const int st = it & 1;
          const uint32_t sq = smem_u32(Qs + st * TB), sd = smem_u32(dOs + st * TB);
          mbar_wait_bounded(&qd_full[st], (it >> 1) & 1, abort_flag, err);
          if (it > 0) mbar_wait_bounded(mma_done, (it - 1) & 1, abort_flag, err);
          tc_fence_after();
#pragma unroll
          for (int kc = 0; kc < D / 16; ++kc) tc_mma_f16(tmem + C::S_COL, kdesc(sk, kc), kdesc(sq, kc), idesc_s, kc > 0);
#pragma unroll
          for (int kc = 0; kc < D / 16; ++kc) tc_mma_f16(tmem + C::DP_COL, kdesc(sv, kc), kdesc(sd, kc), idesc_s, kc > 0);
          tc_commit(s_full);
          mbar_wait_bounded(p_full, it & 1, abort_flag, err);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < TQ / 16; ++kk)
            tc_mma_f16_ts(tmem + C::ACC0, tmem + C::S_COL + kk * 8, mndesc(sd, kk), idesc_a, (it > 0 || kk > 0));
#pragma unroll
          for (int kk = 0; kk < TQ / 16; ++kk)
            tc_mma_f16_ts(tmem + C::ACC1, tmem + C::DP_COL + kk * 8, mndesc(sq, kk), idesc_a, (it > 0 || kk > 0));
          tc_commit(&qd_empty[st]);
          tc_commit(mma_done);
          ++it;
        }
    }
  } else {
    // ------------------------------------------------------ thread = key row
    const int r = warp * 32 + lane;
    const int k = j * TK + r;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    int it = 0;
    for (int hh = 0; hh < hper; ++hh)
      for (int i = 0; i < nqt; ++i) {
        if (!q_seen(i)) continue;
        const int h = h0 + hh;
        // the query tile's lse (log2 units) and delta, staged for every key row
        asm volatile("bar.sync 1, 128;" ::: "memory");
        {
          const int q = i * TQ + r;
          lsm[r] = q < s.S ? lse[(static_cast<long long>(b) * s.hq + h) * s.S + q] * LOG2E_F : 0.f;
          dsm[r] = q < s.S ? delta[(static_cast<long long>(row0) + q) * s.hq + h] : 0.f;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        mbar_wait_bounded(s_full, it & 1, abort_flag, err);
        tc_fence_after();
        const bool need_mask = s.pl > 0 || i == j || (i + 1) * TQ > s.S;
        // 32-column chunks, rolled (a whole row of S and dP would not fit in registers)
#pragma unroll 1
        for (int c = 0; c < TQ / 32; ++c) {
          uint32_t sr[32], dr[32];
          tmem_ld32(tmem + lane_base + C::S_COL + c * 32, sr);
          tmem_ld32(tmem + lane_base + C::DP_COL + c * 32, dr);
          tmem_ld_wait();
          uint32_t pw[16], dw[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float pv[2], dv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int qc = c * 32 + e + u;
              float p = exp2_ftz(__uint_as_float(sr[e + u]) * scale_log2 - lsm[qc]);
              if (need_mask) {
                const int q = i * TQ + qc;
                if (q >= s.S || !visible(s, q, k)) p = 0.f;
              }
              pv[u] = p;
              dv[u] = p * (__uint_as_float(dr[e + u]) - dsm[qc]);
            }
            pw[e >> 1] = pack_bf16x2(pv[0], pv[1]);
            dw[e >> 1] = pack_bf16x2(dv[0], dv[1]);
          }
          tmem_st16(tmem + lane_base + C::S_COL + c * 16, pw);
          tmem_st16(tmem + lane_base + C::DP_COL + c * 16, dw);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        ++it;
      }
    if (it > 0) mbar_wait_bounded(mma_done, (it - 1) & 1, abort_flag, err);
    tc_fence_after();
    // epilogue: dK = scale * (dS^T Q) rotated back by the key's RoPE angles, dV = P^T dO, for
    // this key row; columns i0.. and i0 + D/2.. of the head together (the rotation pairs them)
    const long long T = static_cast<long long>(s.B) * s.S;
    const int pos = pk_pos(s, k);
#pragma unroll 1
    for (int i0 = 0; i0 < D / 2; i0 += 16) {
      uint32_t a1[16], a2[16], v1[16], v2[16];
      tmem_ld16(tmem + lane_base + C::ACC1 + i0, a1);  // dK
      tmem_ld16(tmem + lane_base + C::ACC1 + i0 + D / 2, a2);
      tmem_ld16(tmem + lane_base + C::ACC0 + i0, v1);  // dV
      tmem_ld16(tmem + lane_base + C::ACC0 + i0 + D / 2, v2);
      tmem_ld_wait();
      if (k >= s.S) continue;
      float k1[16], k2[16], w1[16], w2[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        k1[e] = it > 0 ? __uint_as_float(a1[e]) * scale : 0.f;
        k2[e] = it > 0 ? __uint_as_float(a2[e]) * scale : 0.f;
        w1[e] = it > 0 ? __uint_as_float(v1[e]) : 0.f;
        w2[e] = it > 0 ? __uint_as_float(v2[e]) : 0.f;
      }
      rope_back16<D>(s, pos, i0, k1, k2);
      if (hsplit == 1) {
        uint16_t* dk = dqkv + (static_cast<long long>(row0) + k) * s.ld_qkv + (s.hq + g) * D + i0;
        uint16_t* dvp = dqkv + (static_cast<long long>(row0) + k) * s.ld_qkv + (s.hq + s.hkv + g) * D + i0;
        store_bf16x16(dk, k1);
        store_bf16x16(dk + D / 2, k2);
        store_bf16x16(dvp, w1);
        store_bf16x16(dvp + D / 2, w2);
      } else {
        const int per_row = s.hkv * 2 * D;
        float* pr = part + (static_cast<long long>(slice) * T + row0 + k) * per_row + g * 2 * D;
        store_f32x16(pr + i0, k1);
        store_f32x16(pr + i0 + D / 2, k2);
        store_f32x16(pr + D + i0, w1);
        store_f32x16(pr + D + i0 + D / 2, w2);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D>
__global__ void __launch_bounds__(FWD_THREADS, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
                          const AttnShape s, const float* __restrict__ lse, const float* __restrict__ delta,
                          uint16_t* __restrict__ dqkv, int* err) {
  using C = BwdCfg<D>;
  constexpr int TB = C::TILE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* Qs = base;
  uint8_t* dOs = base + TB;
  uint8_t* Ks = base + 2 * TB;  // 2 stages
  uint8_t* Vs = base + 4 * TB;  // 2 stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::BAR_OFF);
  uint64_t* q_full = bars;        // 1
  uint64_t* kv_full = bars + 1;   // 2
  uint64_t* kv_empty = bars + 3;  // 2
  uint64_t* s_full = bars + 5;    // 1
  uint64_t* p_full = bars + 6;    // 1
  uint64_t* mma_done = bars + 7;  // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 9);

  // the last query tiles see the most keys: they start first (longest work first on the SMs)
  const int qt = gridDim.x - 1 - blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (s.hq / s.hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntk = (s.S + TK - 1) / TK;
  const int row0 = b * s.S;
  const float scale = 1.f / sqrtf(static_cast<float>(D));
  const float scale_log2 = scale * LOG2E_F;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, SOFTMAX_WARPS);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == TMA_WARP) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, 2 * TB);
      tma_load_3d(Qs, &tq, 0, row0 + qt * TQ, h * (D / 64), q_full);
      tma_load_3d(dOs, &tdo, 0, row0 + qt * TQ, h * (D / 64), q_full);
      int jj = 0;
      for (int j = 0; j < ntk; ++j) {
        if (!kv_needed(s, qt, j)) continue;
        const int st = jj & 1;
        mbar_wait_bounded(&kv_empty[st], ((jj >> 1) & 1) ^ 1u, abort_flag, err);
        mbar_arrive_expect_tx(&kv_full[st], 2 * TB);
        tma_load_3d(Ks + st * TB, &tq, 0, row0 + j * TK, (s.hq + g) * (D / 64), &kv_full[st]);
        tma_load_3d(Vs + st * TB, &tq, 0, row0 + j * TK, (s.hq + s.hkv + g) * (D / 64), &kv_full[st]);
        ++jj;
      }
    }
  } else if (warp == MMA_WARP) {
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16(TQ, TK, false, false);  // [query, key], K = d
      const uint32_t idesc_q = idesc_bf16(TQ, D, false, true);    // [query, d], K = keys
      const uint32_t sq = smem_u32(Qs), sd = smem_u32(dOs);
      mbar_wait_bounded(q_full, 0, abort_flag, err);
      int jj = 0;
      for (int j = 0; j < ntk; ++j) {
        if (!kv_needed(s, qt, j)) continue;
        const int st = jj & 1;
        const uint32_t sk = smem_u32(Ks + st * TB), sv = smem_u32(Vs + st * TB);
        mbar_wait_bounded(&kv_full[st], (jj >> 1) & 1, abort_flag, err);
        if (jj > 0) mbar_wait_bounded(mma_done, (jj - 1) & 1, abort_flag, err);
        tc_fence_after();
#pragma unroll
        for (int kc = 0; kc < D / 16; ++kc) tc_mma_f16(tmem + C::S_COL, kdesc(sq, kc), kdesc(sk, kc), idesc_s, kc > 0);
#pragma unroll
        for (int kc = 0; kc < D / 16; ++kc) tc_mma_f16(tmem + C::DP_COL, kdesc(sd, kc), kdesc(sv, kc), idesc_s, kc > 0);
        tc_commit(s_full);
        mbar_wait_bounded(p_full, jj & 1, abort_flag, err);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < TK / 16; ++kk)
          tc_mma_f16_ts(tmem + C::ACC0, tmem + C::S_COL + kk * 8, mndesc(sk, kk), idesc_q, (jj > 0 || kk > 0));
        tc_commit(&kv_empty[st]);
        tc_commit(mma_done);
        ++jj;
      }
    }
  } else {
    // ------------------------------------------------------ thread = query row
    const int r = warp * 32 + lane;
    const int q = qt * TQ + r;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float lse2 = q < s.S ? lse[(static_cast<long long>(b) * s.hq + h) * s.S + q] * LOG2E_F : 0.f;
    const float dl = q < s.S ? delta[(static_cast<long long>(row0) + q) * s.hq + h] : 0.f;
    int jj = 0;
    for (int j = 0; j < ntk; ++j) {
      if (!kv_needed(s, qt, j)) continue;
      mbar_wait_bounded(s_full, jj & 1, abort_flag, err);
      tc_fence_after();
      const bool need_mask = s.pl > 0 || j == qt || (j + 1) * TK > s.S;
      // 32-column chunks, rolled (a whole row of S and dP would not fit in registers)
#pragma unroll 1
      for (int c = 0; c < TK / 32; ++c) {
        uint32_t sr[32], dr[32];
        tmem_ld32(tmem + lane_base + C::S_COL + c * 32, sr);
        tmem_ld32(tmem + lane_base + C::DP_COL + c * 32, dr);
        tmem_ld_wait();
        uint32_t dw[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float dv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            float p = exp2_ftz(__uint_as_float(sr[e + u]) * scale_log2 - lse2);
            if (need_mask) {
              const int k = j * TK + c * 32 + e + u;
              if (k >= s.S || !visible(s, q, k)) p = 0.f;
            }
            dv[u] = p * (__uint_as_float(dr[e + u]) - dl);
          }
          dw[e >> 1] = pack_bf16x2(dv[0], dv[1]);
        }
        tmem_st16(tmem + lane_base + C::S_COL + c * 16, dw);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      ++jj;
    }
    if (jj > 0) mbar_wait_bounded(mma_done, (jj - 1) & 1, abort_flag, err);
    tc_fence_after();
    // dQ = scale * (dS K), rotated back by the query's RoPE angles
    uint16_t* qrow = dqkv + (static_cast<long long>(row0) + q) * s.ld_qkv + h * D;
    const int pos = pk_pos(s, q);
#pragma unroll 1
    for (int i0 = 0; i0 < D / 2; i0 += 16) {
      uint32_t a1[16], a2[16];
      tmem_ld16(tmem + lane_base + C::ACC0 + i0, a1);
      tmem_ld16(tmem + lane_base + C::ACC0 + i0 + D / 2, a2);
      tmem_ld_wait();
      if (q >= s.S) continue;
      float f1[16], f2[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        f1[e] = jj > 0 ? __uint_as_float(a1[e]) * scale : 0.f;
        f2[e] = jj > 0 ? __uint_as_float(a2[e]) * scale : 0.f;
      }
      rope_back16<D>(s, pos, i0, f1, f2);
      store_bf16x16(qrow + i0, f1);
      store_bf16x16(qrow + i0 + D / 2, f2);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D>
cudaError_t launch_bwd(const AttnShape& s, const uint16_t* qkv, const uint16_t* o, const uint16_t* dout,
                       const float* lse, float* delta, uint16_t* dqkv, float* ws, size_t ws_bytes, int* err,
                       cudaStream_t st) {
  using C = BwdCfg<D>;
  CUtensorMap tq, tdo;
  const unsigned long long rows = static_cast<unsigned long long>(s.B) * s.S;
  if (!tma_encode_bf16_sw128_planes(&tq, qkv, rows, static_cast<unsigned long long>(s.hq + 2 * s.hkv) * (D / 64),
                                    static_cast<unsigned long long>(s.ld_qkv) * 2, 128, D / 64) ||
      !tma_encode_bf16_sw128_planes(&tdo, dout, rows, static_cast<unsigned long long>(s.hq) * (D / 64),
                                    static_cast<unsigned long long>(s.hq) * D * 2, 128, D / 64))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e =
        cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dq_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int T = s.B * s.S;
  cudaError_t e = attn_delta_launch(o, dout, T, s.hq, D, delta, st);
  if (e != cudaSuccess) return e;
  // head slices: the largest divisor of the group size that keeps the grid within two CTAs per
  // SM and whose fp32 partials fit the workspace
  const int nkt = (s.S + TK - 1) / TK;
  const long long base = static_cast<long long>(nkt) * s.hkv * s.B;
  const int grp = s.hq / s.hkv;
  const size_t per_slice = static_cast<size_t>(T) * s.hkv * 2 * D * sizeof(float);
  int hsplit = 1;
  for (int c = grp; c > 1; --c)
    if (grp % c == 0 && base * c <= 2 * 148 && ws && static_cast<size_t>(c) * per_slice <= ws_bytes) {
      hsplit = c;
      break;
    }
  attn_bwd_dkdv_tc_kernel<D><<<dim3(nkt, s.hkv * hsplit, s.B), FWD_THREADS, C::SMEM_BYTES, st>>>(
      tq, tdo, s, lse, delta, dqkv, hsplit, ws, err);
  g_kernel_launches += 1;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (hsplit > 1) {
    e = attn_dkdv_sum_launch(s, hsplit, ws, dqkv, st);
    if (e != cudaSuccess) return e;
  }
  attn_bwd_dq_tc_kernel<D><<<dim3((s.S + TQ - 1) / TQ, s.hq, s.B), FWD_THREADS, C::SMEM_BYTES, st>>>(tq, tdo, s, lse,
                                                                                                   delta, dqkv, err);
  ++g_kernel_launches;
  return cudaGetLastError();
}

}  // namespace

cudaError_t attn_fwd_launch(const AttnShape& s, const uint16_t* qkv, uint16_t* o, float* lse, int* err,
                               cudaStream_t st) {
  if (s.B <= 0 || s.S <= 0) return cudaSuccess;
  if (s.hq % s.hkv != 0 || (s.pl > 0 && (s.pl + 2 * s.rl != s.S))) return cudaErrorInvalidValue;
  if (s.ld_qkv % 8 != 0) return cudaErrorInvalidValue;
  cudaError_t e;
  if (s.d == 128)
    e = launch_fwd<128>(s, qkv, o, lse, err, st);
  else if (s.d == 64)
    e = launch_fwd<64>(s, qkv, o, lse, err, st);
  else
    return cudaErrorInvalidValue;
  ++g_kernel_launches;
  return e;
}

cudaError_t attn_bwd_launch(const AttnShape& s, const uint16_t* qkv, const uint16_t* o, const uint16_t* dout,
                               const float* lse, float* delta, uint16_t* dqkv, float* ws, size_t ws_bytes, int* err,
                               cudaStream_t st) {
  if (s.B <= 0 || s.S <= 0) return cudaSuccess;
  if (s.hkv <= 0 || s.hq % s.hkv != 0 || (s.pl > 0 && (s.pl + 2 * s.rl != s.S))) return cudaErrorInvalidValue;
  if (s.ld_qkv % 8 != 0 || (ws && (reinterpret_cast<uintptr_t>(ws) & 15u))) return cudaErrorInvalidValue;
  if (s.d == 128) return launch_bwd<128>(s, qkv, o, dout, lse, delta, dqkv, ws, ws_bytes, err, st);
  if (s.d == 64) return launch_bwd<64>(s, qkv, o, dout, lse, delta, dqkv, ws, ws_bytes, err, st);
  return cudaErrorInvalidValue;
}

cudaError_t attn_delta_launch(const uint16_t* o, const uint16_t* dout, int T, int hq, int d, float* delta,
                              cudaStream_t st) {
  const long long warps = static_cast<long long>(T) * hq;
  attn_delta_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, st>>>(o, dout, T, hq, d, delta);
  ++g_kernel_launches;
  return cudaGetLastError();
}

cudaError_t attn_dkdv_sum_launch(const AttnShape& s, int hsplit, const float* part, uint16_t* dqkv, cudaStream_t st) {
  const long long n4 = static_cast<long long>(s.B) * s.S * s.hkv * 2 * s.d / 4;
  attn_dkdv_sum_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, st>>>(s, hsplit, part, dqkv);
  ++g_kernel_launches;
  return cudaGetLastError();
}

}  // namespace soup
