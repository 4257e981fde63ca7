// Tensor-core GEMM for sm_100a: C[M,N] = sum over segments of A_s[M,K_s] . B_s[N,K_s]^T.
//
// This single kernel carries every contraction of the decoder layer:
//   * forward  y = x W^T + s (x A^T) B^T : segment 0 streams the NF4 weight (dequantised by the
//     producer warps), later segments are the LoRA branch appended as extra K-blocks;
//   * backward dx = dy W + s (dy B) A     : the same NF4 weight read transposed;
//   * LoRA grads, lm_head forward/backward: plain bf16 / fp32 operands.
//
// Roles (512 threads, one CTA per (MT*128) x BN output tile, or per K-slice of it under split-K):
//   warps 0-11  producers, three groups of four warps that take alternate k-blocks.  On the NF4
//               path each dequantises one B tile from raw codes / q8 absmax staged by TMA
//               (per-absmax-block table of bf16 products in registers, byte-permute lookups)
//               into the 128-byte-swizzled layout the MMA reads; other operands the TMA does
//               not carry are gathered and converted here;
//   warp 12     allocates TMEM; lane 0 issues tcgen05.mma (M=128 per half, N=BN, K=16) and
//               tcgen05.commit to release stages;
//   warp 13     lane 0 issues the operand TMA loads (A, bf16 B) into the stage ring;
//   warp 14     lane 0 issues the raw NF4 TMA loads into a ring of their own, so they run
//               ahead of the operand stages (a raw slot frees when its k-block is decoded);
//   warps 12-15 epilogue: tcgen05.ld rows out of TMEM, scale, add residual / old value, store
//               (under split-K: store an fp32 partial tile; the tile's last split to finish
//               sums all partials in split order and runs the normal epilogue).
//
// NF4 decode follows the double-quantised format: mhat = fp32(fp32(q8 * s2) + mean),
// w = bf16_rn(fp32(code_value * mhat)), one float32 multiply per element.
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>

namespace soup {

namespace {

constexpr int GROUPS = 3;                       // producer groups (4 warps each) on alternate k-blocks
constexpr int PRODUCER_WARPS = 4 * GROUPS;
constexpr int EPI_WARP0 = PRODUCER_WARPS;       // first of the 4 epilogue warps (a whole warpgroup)
constexpr int GEMM_THREADS = 32 * (PRODUCER_WARPS + 4);
constexpr int GROUP_THREADS = 128;
constexpr int UM = 128;  // rows of one tcgen05.mma (cta_group::1); a CTA tile stacks MT of them
constexpr int BK = 64;   // 64 bf16 = 128 bytes = one swizzle row
constexpr int SMEM_LIMIT = 232448;  // 227 KiB of dynamic shared memory per CTA

template <int MT, int BN>
struct GemmCfg {
  static constexpr int BM = UM * MT;
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // one k-block of both MMA operands
  // Raw NF4 staging (TMA) in a ring of its own: codes BN x 32 B (forward) or 64 x BN/2 B
  // (transposed), q8 absmax BN x 16 B or 64 x 16 B.  A raw slot is released as soon as its
  // k-block is dequantised, so the raw loads run several k-blocks ahead of the operand stages.
  // (Batching four k-blocks of codes per copy, with the q8 bytes loaded by the producers,
  // measured 5-13 % slower on the 8B projection shapes at 512 rows.)
  static constexpr int RAW_CODE_BYTES = BN * 32;
  static constexpr int RAW_Q8_BYTES = (BN > 64 ? BN : 64) * 16;
  static constexpr int RAW_BYTES = RAW_CODE_BYTES + RAW_Q8_BYTES;
  // Every operand stage comes with at least one raw slot (RAW_SLOTS >= STAGES): a producer that
  // waits for raw k-block kb has seen the MMAs of kb - STAGES retire, so every raw k-block up
  // to kb - STAGES has landed and been decoded; with RAW_SLOTS >= STAGES that covers kb -
  // RAW_SLOTS, the previous use of kb's slot, and the slot's parity wait cannot alias it.
  // (With more stages than raw slots only the order in which TMA loads complete keeps the
  // phases apart.)
  static constexpr int CTRL_BYTES = 640;
  static constexpr int AVAIL = SMEM_LIMIT - 1024 - CTRL_BYTES;
  static constexpr int STAGES_FIT = AVAIL / (STAGE_BYTES + RAW_BYTES);
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int RAW_FIT = (AVAIL - STAGES * STAGE_BYTES) / RAW_BYTES;
  static constexpr int RAW_SLOTS = RAW_FIT > 16 ? 16 : RAW_FIT;
  static constexpr int TMEM_COLS = MT * BN;  // one BN-column fp32 accumulator per 128-row half
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + RAW_SLOTS * RAW_BYTES + CTRL_BYTES;
};

// Instruction descriptor of the GEMM's MMAs: M = 128 rows, N = BN.
template <int BN>
__device__ __forceinline__ uint32_t idesc_bf16_f32(bool a_mn_major, bool b_mn_major) {
  return idesc_bf16(UM, BN, a_mn_major, b_mn_major);
}

// ---------------------------------------------------------------- operand fetch
__device__ __forceinline__ int nf4_seg_of(const NF4Group& g, int wr) {
  int s = 0;
  if (g.nseg > 1 && wr >= g.seg[1].row_begin) s = 1;
  if (g.nseg > 2 && wr >= g.seg[2].row_begin) s = 2;
  return s;
}

// Raw gather of one NF4 chunk (8 consecutive columns of W row wr): code word, q8, s2, segment.
struct NF4Raw {
  uint32_t code;
  float s2;
  int q8;
  int seg;
};
__device__ __forceinline__ NF4Raw nf4_gather(const NF4Group& g, int wr, int wc) {
  const int s = nf4_seg_of(g, wr);
  const NF4Seg& sg = g.seg[s];
  const long long flat = static_cast<long long>(wr - sg.row_begin) * g.cols + wc;
  const long long blk = flat >> 6;
  NF4Raw r;
  r.code = __ldg(reinterpret_cast<const uint32_t*>(sg.codes + (flat >> 1)));
  r.q8 = __ldg(sg.q8 + blk);
  r.s2 = __ldg(sg.scales + (blk >> 8));
  r.seg = s;
  return r;
}
__device__ __forceinline__ uint4 nf4_decode(const NF4Raw& r, const float* lut, const float* seg_mean) {
  const float mh = __fadd_rn(__fmul_rn(static_cast<float>(r.q8), r.s2), seg_mean[r.seg]);
  const uint32_t c = r.code;
  uint4 o;
  o.x = pack_bf16x2(__fmul_rn(lut[c & 15u], mh), __fmul_rn(lut[(c >> 4) & 15u], mh));
  o.y = pack_bf16x2(__fmul_rn(lut[(c >> 8) & 15u], mh), __fmul_rn(lut[(c >> 12) & 15u], mh));
  o.z = pack_bf16x2(__fmul_rn(lut[(c >> 16) & 15u], mh), __fmul_rn(lut[(c >> 20) & 15u], mh));
  o.w = pack_bf16x2(__fmul_rn(lut[(c >> 24) & 15u], mh), __fmul_rn(lut[c >> 28], mh));
  return o;
}

__device__ __forceinline__ uint4 cvt_f32x8(const float* src, float s) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(src)), b = __ldg(reinterpret_cast<const float4*>(src) + 1);
  uint4 o;
  o.x = pack_bf16x2(a.x * s, a.y * s);
  o.y = pack_bf16x2(a.z * s, a.w * s);
  o.z = pack_bf16x2(b.x * s, b.y * s);
  o.w = pack_bf16x2(b.z * s, b.w * s);
  return o;
}

// 8 consecutive k of row r (K-major, non-NF4 kinds).
__device__ __forceinline__ uint4 fetch_kmajor(const Operand& op, int r, int k) {
  if (op.kind == OP_BF16_K)
    return __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(op.ptr) + r * op.ld + k));
  return cvt_f32x8(static_cast<const float*>(op.ptr) + r * op.ld + k, op.scale);  // OP_F32_K
}
// 8 consecutive rows [r, r+8) at reduction index k (MN-major, non-NF4 kinds), zero past K.
__device__ __forceinline__ uint4 fetch_mn8(const Operand& op, int r, int k, int K) {
  if (k >= K) return make_uint4(0, 0, 0, 0);
  if (op.kind == OP_BF16_MN)
    return __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(op.ptr) + k * op.ld + r));
  return cvt_f32x8(static_cast<const float*>(op.ptr) + k * op.ld + r, op.scale);  // OP_F32_MN
}

__device__ __forceinline__ uint32_t swz_off(int r, int chunk) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((chunk ^ (r & 7)) << 4));
}

__device__ __forceinline__ void store_mn_pairs(uint8_t* tile, int rr0, int kp, const uint4& x0, const uint4& x1) {
  const uint32_t a[4] = {x0.x, x0.y, x0.z, x0.w};
  const uint32_t b[4] = {x1.x, x1.y, x1.z, x1.w};
  const uint32_t inchunk = (kp & 3) * 4;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t lo = __byte_perm(a[j], b[j], 0x5410);  // row 2j:   (k, k+1)
    const uint32_t hi = __byte_perm(a[j], b[j], 0x7632);  // row 2j+1: (k, k+1)
    *reinterpret_cast<uint32_t*>(tile + swz_off(rr0 + 2 * j, kp >> 2) + inchunk) = lo;
    *reinterpret_cast<uint32_t*>(tile + swz_off(rr0 + 2 * j + 1, kp >> 2) + inchunk) = hi;
  }
}

// Fill one ROWS x 64 tile of an operand (group-cooperative, gtid in [0, 128)).
template <int ROWS>
__device__ __forceinline__ void load_tile(const Operand& op, const NF4Group& g, const float* lut,
                                          const float* seg_mean, int K, int row0, int nrows, int k0, uint8_t* tile,
                                          int gtid) {
  if (op.kind == OP_NF4_K) {
    constexpr int CH = ROWS * 8 / GROUP_THREADS;
    constexpr int BATCH = CH < 4 ? CH : 4;  // chunks gathered before any is decoded
#pragma unroll
    for (int b0 = 0; b0 < CH; b0 += BATCH) {
      NF4Raw raw[BATCH];
      bool ok[BATCH];
#pragma unroll
      for (int i = 0; i < BATCH; ++i) {  // phase 1: issue the global loads of the batch
        const int c = gtid + (b0 + i) * GROUP_THREADS;
        const int row = row0 + (c >> 3), k = k0 + (c & 7) * 8;
        ok[i] = row < nrows && row >= op.row_lo && row < op.row_hi && k < K;
        if (ok[i]) raw[i] = nf4_gather(g, row, k);
      }
#pragma unroll
      for (int i = 0; i < BATCH; ++i) {  // phase 2: dequantise and store
        const int c = gtid + (b0 + i) * GROUP_THREADS;
        const uint4 v = ok[i] ? nf4_decode(raw[i], lut, seg_mean) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(tile + swz_off(c >> 3, c & 7)) = v;
      }
    }
  } else if (op.kind == OP_NF4_MN) {
    constexpr int U = (ROWS / 8) * 32 / GROUP_THREADS;
    constexpr int BATCH = U < 2 ? U : 2;
#pragma unroll
    for (int b0 = 0; b0 < U; b0 += BATCH) {
      NF4Raw r0[BATCH], r1[BATCH];
      bool ok0[BATCH], ok1[BATCH];
#pragma unroll
      for (int i = 0; i < BATCH; ++i) {
        const int u = gtid + (b0 + i) * GROUP_THREADS;
        const int kp = u & 31, row = row0 + (u >> 5) * 8, k = k0 + kp * 2;
        const bool rows_ok = row < nrows;
        ok0[i] = rows_ok && k < K;
        ok1[i] = rows_ok && k + 1 < K;
        if (ok0[i]) r0[i] = nf4_gather(g, k, row);
        if (ok1[i]) r1[i] = nf4_gather(g, k + 1, row);
      }
#pragma unroll
      for (int i = 0; i < BATCH; ++i) {
        const int u = gtid + (b0 + i) * GROUP_THREADS;
        const uint4 x0 = ok0[i] ? nf4_decode(r0[i], lut, seg_mean) : make_uint4(0, 0, 0, 0);
        const uint4 x1 = ok1[i] ? nf4_decode(r1[i], lut, seg_mean) : make_uint4(0, 0, 0, 0);
        store_mn_pairs(tile, (u >> 5) * 8, u & 31, x0, x1);
      }
    }
  } else if (op.kind == OP_BF16_K || op.kind == OP_F32_K) {
#pragma unroll 4
    for (int c = gtid; c < ROWS * 8; c += GROUP_THREADS) {
      const int rr = c >> 3, kc = c & 7;
      const int row = row0 + rr, k = k0 + kc * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (row < nrows && row >= op.row_lo && row < op.row_hi && k < K) v = fetch_kmajor(op, row, k);
      *reinterpret_cast<uint4*>(tile + swz_off(rr, kc)) = v;
    }
  } else {  // OP_BF16_MN / OP_F32_MN: units of 8 rows x 2 consecutive k
#pragma unroll 2
    for (int u = gtid; u < (ROWS / 8) * 32; u += GROUP_THREADS) {
      const int kp = u & 31, rr0 = (u >> 5) * 8;
      const int row = row0 + rr0, k = k0 + kp * 2;
      uint4 x0 = make_uint4(0, 0, 0, 0), x1 = make_uint4(0, 0, 0, 0);
      if (row < nrows && row >= op.row_lo && row < op.row_hi) {
        x0 = fetch_mn8(op, row, k, K);
        x1 = fetch_mn8(op, row, k + 1, K);
      }
      store_mn_pairs(tile, rr0, kp, x0, x1);
    }
  }
}

// Explicit shared-space accesses for the decode path (32-bit shared addresses).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ int lds_s8(uint32_t a) {
  int v;
  asm volatile("ld.shared.s8 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t a, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// PTX byte permute in its default mode: each selector nibble's low 3 bits pick one of the 8
// source bytes; a set bit 3 replicates that byte's sign bit over the result byte.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Per-block decode table: the 16 values bf16_rn(codebook[j] * mh) of one absmax block, kept as
// 4 words of low bytes (L) and 4 words of high bytes (H), entry j in byte j%4 of word j/4.
struct BlockLut {
  uint32_t L[4], H[4];
};
__device__ __forceinline__ BlockLut block_lut(const float (&cb)[16], float mh) {
  uint32_t R[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) R[i] = pack_bf16x2(__fmul_rn(cb[2 * i], mh), __fmul_rn(cb[2 * i + 1], mh));
  BlockLut t;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    t.L[i] = prmt(R[2 * i], R[2 * i + 1], 0x6420);
    t.H[i] = prmt(R[2 * i], R[2 * i + 1], 0x7531);
  }
  return t;
}
// Four table lookups with byte permutes: s holds four 3-bit indices (nibbles), m has 0xFF in
// the bytes whose code is >= 8 (upper half of the table).  Returns two bf16x2 words.
__device__ __forceinline__ void lut4(const BlockLut& t, uint32_t s, uint32_t m, uint32_t& o01, uint32_t& o23) {
  const uint32_t lo = (prmt(t.L[0], t.L[1], s) & ~m) | (prmt(t.L[2], t.L[3], s) & m);
  const uint32_t hi = (prmt(t.H[0], t.H[1], s) & ~m) | (prmt(t.H[2], t.H[3], s) & m);
  o01 = prmt(lo, hi, 0x5140);
  o23 = prmt(lo, hi, 0x7362);
}
// The 8 codes of one 32-bit word (element 2i = low nibble of byte i) through the block table.
__device__ __forceinline__ uint4 decode_word_lut(uint32_t c, const BlockLut& t) {
  const uint32_t c4 = c << 4;
  const uint32_t m0 = prmt(c4, c, 0xD9C8);  // sign-replicated bit 3 of nibbles 0..3
  const uint32_t m1 = prmt(c4, c, 0xFBEA);  // ... of nibbles 4..7
  uint4 o;
  lut4(t, c & 0x7777u, m0, o.x, o.y);
  lut4(t, (c >> 16) & 0x7777u, m1, o.z, o.w);
  return o;
}

// Dequantise the forward (W[n, k]) B tile from TMA-staged raw codes / q8 absmax.
// raw_codes: [BN][32] bytes (row n, k0..k0+63 = exactly one absmax block); raw_q8: [BN][16]
// bytes covering k-blocks [16*floor(kbw/16), +16) of each row; the tile lies inside NF4
// tensor `s`.  One thread decodes a whole 64-element row block (one absmax, 8 stores).
// Group scales (s2) of the absmax blocks a thread decodes in one k-block, loaded before the
// thread waits for the raw tile so their latency overlaps the wait.
template <int BN>
__device__ __forceinline__ void fwd_scales(const NF4Group& g, int s, int n0, int N, int kbw, int gtid, float* s2) {
  const NF4Seg& sg = g.seg[s];
  const long long cpr = g.cols >> 6;
#pragma unroll
  for (int i = 0; i < (BN + GROUP_THREADS - 1) / GROUP_THREADS; ++i) {
    const int r = gtid + i * GROUP_THREADS;
    s2[i] = 0.f;
    if (r < BN && n0 + r < N) {
      const long long blk = static_cast<long long>(n0 + r - sg.row_begin) * cpr + kbw;
      s2[i] = __ldg(sg.scales + (blk >> 8));
    }
  }
}
template <int BN>
__device__ __forceinline__ void dx_scales(const NF4Group& g, int s, int n0, int N, int k0, int gtid, float* s2) {
  const NF4Seg& sg = g.seg[s];
  const long long cpr = g.cols >> 6;
  constexpr int NB = BN / 64;
#pragma unroll
  for (int i = 0; i < (64 * NB + GROUP_THREADS - 1) / GROUP_THREADS; ++i) {
    const int u = gtid + i * GROUP_THREADS;
    s2[i] = 0.f;
    const int kr = u / NB, b = u % NB;
    if (u < 64 * NB && n0 + b * 64 < N) {
      const long long blk = static_cast<long long>(k0 + kr - sg.row_begin) * cpr + ((n0 + b * 64) >> 6);
      s2[i] = __ldg(sg.scales + (blk >> 8));
    }
  }
}

template <int BN>
__device__ __forceinline__ void decode_fwd_raw(const NF4Group& g, int s, const float (&cb)[16], const float* seg_mean,
                                               int n0, int N, int kbw, const uint8_t* raw_codes,
                                               const uint8_t* raw_q8, uint8_t* tile, int gtid, const float* s2) {
  const float mean = seg_mean[s];
#pragma unroll
  for (int i = 0; i < (BN + GROUP_THREADS - 1) / GROUP_THREADS; ++i) {
    const int r = gtid + i * GROUP_THREADS;
    if (r >= BN) break;
    const uint32_t trow = smem_u32(tile) + (r >> 3) * 1024 + (r & 7) * 128;
    if (n0 + r < N) {
      const uint32_t rc = smem_u32(raw_codes) + r * 32;
      const uint4 w0 = lds128(rc);
      const uint4 w1 = lds128(rc + 16);
      const int q8 = lds_s8(smem_u32(raw_q8) + r * 16 + (kbw & 15));
      const float mh = __fadd_rn(__fmul_rn(static_cast<float>(q8), s2[i]), mean);
      const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      const BlockLut t = block_lut(cb, mh);
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) sts128(trow + ((kc ^ (r & 7)) << 4), decode_word_lut(words[kc], t));
    } else {
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) sts128(trow + ((kc ^ (r & 7)) << 4), make_uint4(0, 0, 0, 0));
    }
  }
}

// Dequantise the transposed (dX) B tile: B[n, k] = W[k0 + k, n0 + n] from raw codes
// [64][BN/2] bytes and raw q8 [64][16] bytes (absmax blocks [xq, xq+16) of each W row), into
// the MN-major 128-byte-swizzled layout.  One thread decodes one absmax block: 64
// consecutive n of one k (= one 128-byte swizzle row, 8 conflict-free 16-byte stores).
template <int BN>
__device__ __forceinline__ void decode_dx_raw(const NF4Group& g, int s, const float (&cb)[16], const float* seg_mean,
                                              int n0, int N, int k0, int xq, const uint8_t* raw_codes,
                                              const uint8_t* raw_q8, uint8_t* tile, int gtid, const float* s2) {
  constexpr int NB = BN / 64;  // absmax blocks per W row in the tile
  const float mean = seg_mean[s];
#pragma unroll
  for (int i = 0; i < (64 * NB + GROUP_THREADS - 1) / GROUP_THREADS; ++i) {
    const int u = gtid + i * GROUP_THREADS;
    if (u >= 64 * NB) break;
    const int kr = u / NB, b = u % NB;
    const int n = n0 + b * 64;
    const uint32_t dst = smem_u32(tile) + b * 8192 + (kr >> 3) * 1024 + (kr & 7) * 128;
    if (n < N) {
      const uint32_t rc = smem_u32(raw_codes) + kr * (BN / 2) + b * 32;
      const uint4 w0 = lds128(rc);
      const uint4 w1 = lds128(rc + 16);
      const int bcol = n >> 6;
      const int q8 = lds_s8(smem_u32(raw_q8) + kr * 16 + (bcol - xq));
      const float mh = __fadd_rn(__fmul_rn(static_cast<float>(q8), s2[i]), mean);
      const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      const BlockLut t = block_lut(cb, mh);
#pragma unroll
      for (int nc = 0; nc < 8; ++nc) sts128(dst + ((nc ^ (kr & 7)) << 4), decode_word_lut(words[nc], t));
    } else {
#pragma unroll
      for (int nc = 0; nc < 8; ++nc) sts128(dst + ((nc ^ (kr & 7)) << 4), make_uint4(0, 0, 0, 0));
    }
  }
}

__device__ __forceinline__ bool seg_active(const GemmSeg& s, int n0, int bn) {
  if (s.K <= 0) return false;
  return s.B.row_lo < n0 + bn && s.B.row_hi > n0;
}

// Epilogue store of NC consecutive columns [col0, col0 + NC) of row `row` (values already
// scaled; columns at or past N are skipped, N a multiple of 8).  Every load (residual, the
// old value of an accumulated output) is issued before the first store: a read-modify-write
// written column by column makes each store wait for its own load, so a warp would wait on
// memory once per column instead of once per call.
template <int NC>
__device__ __forceinline__ void epilogue_store(const GemmParams& p, int row, int col0, float (&v)[NC]) {
  static_assert(NC % 8 == 0, "columns come in groups of 8");
  constexpr int G8 = NC / 8;
  const int nv = p.N - col0;  // columns in range (>= 8)
  if (!p.out_trans) {
    if (p.residual) {
      const uint16_t* res = static_cast<const uint16_t*>(p.residual) + row * p.ldr + col0;
      uint4 rv[G8];
#pragma unroll
      for (int g = 0; g < G8; ++g)
        if (g * 8 < nv) rv[g] = *reinterpret_cast<const uint4*>(res + g * 8);
#pragma unroll
      for (int g = 0; g < G8; ++g) {
        if (g * 8 >= nv) break;
        const uint32_t rw[4] = {rv[g].x, rv[g].y, rv[g].z, rv[g].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack_bf16x2(rw[j]);
          v[g * 8 + 2 * j] += f.x;
          v[g * 8 + 2 * j + 1] += f.y;
        }
      }
    }
    if (p.out_f32) {
      float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * p.ldo + col0);
      if (p.accumulate) {
        float4 a[2 * G8];
#pragma unroll
        for (int g = 0; g < 2 * G8; ++g)
          if (g * 4 < nv) a[g] = o[g];
#pragma unroll
        for (int g = 0; g < 2 * G8; ++g) {
          if (g * 4 >= nv) break;
          v[4 * g] += a[g].x; v[4 * g + 1] += a[g].y; v[4 * g + 2] += a[g].z; v[4 * g + 3] += a[g].w;
        }
      }
#pragma unroll
      for (int g = 0; g < 2 * G8; ++g)
        if (g * 4 < nv) o[g] = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
    } else {
      uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * p.ldo + col0);
      if (p.accumulate) {
        uint4 a[G8];
#pragma unroll
        for (int g = 0; g < G8; ++g)
          if (g * 8 < nv) a[g] = o[g];
#pragma unroll
        for (int g = 0; g < G8; ++g) {
          if (g * 8 >= nv) break;
          const uint32_t aw[4] = {a[g].x, a[g].y, a[g].z, a[g].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = unpack_bf16x2(aw[j]);
            v[g * 8 + 2 * j] += f.x;
            v[g * 8 + 2 * j + 1] += f.y;
          }
        }
      }
#pragma unroll
      for (int g = 0; g < G8; ++g)
        if (g * 8 < nv)
          o[g] = make_uint4(pack_bf16x2(v[g * 8], v[g * 8 + 1]), pack_bf16x2(v[g * 8 + 2], v[g * 8 + 3]),
                            pack_bf16x2(v[g * 8 + 4], v[g * 8 + 5]), pack_bf16x2(v[g * 8 + 6], v[g * 8 + 7]));
    }
  } else {
    // transposed output: column c of the tile is row c of `out` (a warp's 32 rows are 32
    // consecutive elements there)
    if (p.out_f32) {
      float* o = static_cast<float*>(p.out) + static_cast<long long>(col0) * p.ldo + row;
      if (p.accumulate) {
        float a[NC];
#pragma unroll
        for (int j = 0; j < NC; ++j)
          if (j < nv) a[j] = o[j * p.ldo];
#pragma unroll
        for (int j = 0; j < NC; ++j) v[j] += (j < nv) ? a[j] : 0.f;
      }
#pragma unroll
      for (int j = 0; j < NC; ++j)
        if (j < nv) o[j * p.ldo] = v[j];
    } else {
      uint16_t* o = static_cast<uint16_t*>(p.out) + static_cast<long long>(col0) * p.ldo + row;
      if (p.accumulate) {
        uint16_t a[NC];
#pragma unroll
        for (int j = 0; j < NC; ++j)
          if (j < nv) a[j] = o[j * p.ldo];
#pragma unroll
        for (int j = 0; j < NC; ++j) v[j] += (j < nv) ? bf16_to_f32(a[j]) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < NC; ++j)
        if (j < nv) {
          const __nv_bfloat16 b = __float2bfloat16_rn(v[j]);
          o[j * p.ldo] = *reinterpret_cast<const uint16_t*>(&b);
        }
    }
  }
}

// RoPE epilogue of one row: a[16] / b[16] are the accumulator columns i0..i0+15 and
// i0 + d/2.. of one head (i0 < d/2) whose first column is col_head; rotated by the row's angles
// (pos * theta^(-2i/d) from the cos / sin tables) after scaling, then rounded to bf16 once.
__device__ __forceinline__ void rope_store16(const GemmParams& p, int row, int col_head, int i0, const uint32_t (&a)[16],
                                             const uint32_t (&b)[16]) {
  const int half = p.rope_d >> 1;
  int pos = row % p.rope_S;
  if (p.rope_rl > 0 && pos >= p.rope_S - p.rope_rl) pos -= p.rope_rl;
  const float4* cp = reinterpret_cast<const float4*>(p.rope_cos + static_cast<long long>(pos) * half + i0);
  const float4* sp = reinterpret_cast<const float4*>(p.rope_sin + static_cast<long long>(pos) * half + i0);
  float c[16], sn[16];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const float4 cv = __ldg(cp + g), sv = __ldg(sp + g);
    c[4 * g] = cv.x; c[4 * g + 1] = cv.y; c[4 * g + 2] = cv.z; c[4 * g + 3] = cv.w;
    sn[4 * g] = sv.x; sn[4 * g + 1] = sv.y; sn[4 * g + 2] = sv.z; sn[4 * g + 3] = sv.w;
  }
  uint32_t w1[8], w2[8];
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    float o1[2], o2[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float x1 = p.alpha * __uint_as_float(a[j + u]), x2 = p.alpha * __uint_as_float(b[j + u]);
      o1[u] = x1 * c[j + u] - x2 * sn[j + u];
      o2[u] = x2 * c[j + u] + x1 * sn[j + u];
    }
    w1[j >> 1] = pack_bf16x2(o1[0], o1[1]);
    w2[j >> 1] = pack_bf16x2(o2[0], o2[1]);
  }
  uint16_t* o = static_cast<uint16_t*>(p.out) + static_cast<long long>(row) * p.ldo + col_head + i0;
  reinterpret_cast<uint4*>(o)[0] = make_uint4(w1[0], w1[1], w1[2], w1[3]);
  reinterpret_cast<uint4*>(o)[1] = make_uint4(w1[4], w1[5], w1[6], w1[7]);
  reinterpret_cast<uint4*>(o + half)[0] = make_uint4(w2[0], w2[1], w2[2], w2[3]);
  reinterpret_cast<uint4*>(o + half)[1] = make_uint4(w2[4], w2[5], w2[6], w2[7]);
}

// Group-scale registers of one k-block of the NF4 B tile (forward: one per row this thread
// decodes; dX: one per absmax block).
template <int BN>
struct ScaleRegs {
  static constexpr int NF = (BN + GROUP_THREADS - 1) / GROUP_THREADS;
  static constexpr int ND = (64 * (BN / 64) + GROUP_THREADS - 1) / GROUP_THREADS;
  static constexpr int N = NF > ND ? NF : ND;
  float v[N];
};
template <int BN>
__device__ __forceinline__ void load_scales(const GemmParams& p, bool fwd, int n0, int kk, int gtid, ScaleRegs<BN>& r) {
  if (fwd)
    fwd_scales<BN>(p.nf4, nf4_seg_of(p.nf4, n0), n0, p.N, kk, gtid, r.v);
  else
    dx_scales<BN>(p.nf4, nf4_seg_of(p.nf4, kk * BK), n0, p.N, kk * BK, gtid, r.v);
}

// ---------------------------------------------------------------- work pieces
// A CTA's work is a list of pieces: an output tile and a range [kb_lo, kb_hi) of its k-blocks
// (the active segments' k-blocks concatenated).  Without stream-K: one piece, the tile of
// (blockIdx.x, blockIdx.y) and split blockIdx.z of `splits`.  With stream-K: the k-blocks of
// all tiles, flattened tile by tile (M-tiles fastest), are cut into sk_ctas equal ranges, one
// per CTA; a range holds the tail of one tile, whole tiles, then the head of another.  A tile
// cut between CTAs is partial: each CTA stores its fp32 share in a workspace slot (slot 2c for
// CTA c's first piece, 2c + 1 for its last) and the CTA that completes the tile's count sums
// the shares in k order at its end.
struct Piece {
  int m0, n0, kb_lo, kb_hi, tile;
  int partial;  // the tile's k-blocks are shared with other CTAs (or other splits)
};
template <bool SK>
__device__ __forceinline__ int piece_count(const GemmParams& p) {
  if (!SK) return 1;
  return sk_piece_count(p.sk_tiles, p.sk_nkt, p.sk_ctas, blockIdx.x);
}
template <int BM, int BN, bool SK>
__device__ __forceinline__ Piece piece_at(const GemmParams& p, int pc) {
  Piece z;
  if (!SK) {
    z.n0 = blockIdx.x * BN;
    z.m0 = blockIdx.y * BM;
    z.tile = blockIdx.y * gridDim.x + blockIdx.x;
    int nkb_all = 0;
    for (int s = 0; s < p.nseg; ++s)
      if (seg_active(p.seg[s], z.n0, BN)) nkb_all += (p.seg[s].K + BK - 1) / BK;
    const int splits = p.splits > 1 ? p.splits : 1;
    z.kb_lo = static_cast<int>(static_cast<long long>(blockIdx.z) * nkb_all / splits);
    z.kb_hi = static_cast<int>(static_cast<long long>(blockIdx.z + 1) * nkb_all / splits);
    z.partial = splits > 1 ? 1 : 0;
    return z;
  }
  sk_piece(p.sk_tiles, p.sk_nkt, p.sk_ctas, blockIdx.x, pc, &z.tile, &z.kb_lo, &z.kb_hi);
  z.m0 = (z.tile % p.sk_tiles_m) * BM;
  z.n0 = (z.tile / p.sk_tiles_m) * BN;
  z.partial = (z.kb_lo == 0 && z.kb_hi == p.sk_nkt) ? 0 : 1;
  return z;
}

// ---------------------------------------------------------------- the kernel
// SK: the stream-K form (p.sk_ctas > 0); the whole-tile / split-K form keeps its own
// instantiation, with one piece known at compile time.
template <int MT, int BN, bool SK>
__global__ void __launch_bounds__(GEMM_THREADS, 1) gemm_tc_kernel(const __grid_constant__ GemmParams p) {
  using C = GemmCfg<MT, BN>;
  constexpr int BM = C::BM;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* raw_base = base + C::STAGES * C::STAGE_BYTES;
  uint8_t* ctrl = raw_base + C::RAW_SLOTS * C::RAW_BYTES;
  float* lut = reinterpret_cast<float*>(ctrl);                       // 16 floats
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 64);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl + 68);
  volatile int* last_flag = reinterpret_cast<volatile int*>(ctrl + 72);  // split-K: this CTA reduces
  float* seg_mean = reinterpret_cast<float*>(ctrl + 80);              // up to 3 NF4 tensors
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl + 128);
  uint64_t* empty = full + C::STAGES;
  uint64_t* raw_full = empty + C::STAGES;
  uint64_t* raw_empty = raw_full + C::RAW_SLOTS;
  uint64_t* done = raw_empty + C::RAW_SLOTS;
  uint64_t* tmem_empty = done + 1;  // the epilogue has read the accumulator out of TMEM
  static_assert(128 + 8 * (2 * C::STAGES + 2 * C::RAW_SLOTS + 2) <= C::CTRL_BYTES, "control block overflow");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], GROUP_THREADS / 32 + 1);  // 4 producer warps + the TMA issuer
      mbar_init(&empty[s], 1);
    }
    for (int r = 0; r < C::RAW_SLOTS; ++r) {
      mbar_init(&raw_full[r], 1);
      mbar_init(&raw_empty[r], GROUP_THREADS / 32);  // the 4 warps of the group that decoded it
    }
    mbar_init(done, 1);
    mbar_init(tmem_empty, 4);  // one arrival per epilogue warp
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (threadIdx.x < 16) lut[threadIdx.x] = p.lut[threadIdx.x];
  if (threadIdx.x >= 32 && threadIdx.x < 32 + p.nf4.nseg) seg_mean[threadIdx.x - 32] = *p.nf4.seg[threadIdx.x - 32].mean;
  if (warp == EPI_WARP0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_pieces = piece_count<SK>(p);
  const int splits = p.splits > 1 ? p.splits : 1;

  // Every role walks the same pieces in the same order.  Stage and raw-slot indices (and
  // their phases) run on across pieces: kb_run / raw_run count the k-blocks / raw k-blocks of
  // this CTA's earlier pieces.  Within a piece, raw-staged k-blocks (segment 0 when raw_tma)
  // come first: local k-blocks [0, n_raw).
  if (warp < PRODUCER_WARPS) {
    // ------------------------------------------------ producers (groups on alternate k-blocks)
    const int grp = warp >> 2, gtid = threadIdx.x & (GROUP_THREADS - 1);
    const float(&cb)[16] = p.lut;  // kernel-parameter (constant bank) operands, no registers
    int kb_run = 0, raw_run = 0;
    for (int pc = 0; pc < n_pieces; ++pc) {
      const Piece z = piece_at<BM, BN, SK>(p, pc);
      const int n0 = z.n0, m0 = z.m0, kb_lo = z.kb_lo, kb_hi = z.kb_hi;
      const bool seg0_raw = p.raw_tma && seg_active(p.seg[0], n0, BN);
      const int seg0_nk = seg0_raw ? (p.seg[0].K + BK - 1) / BK : 0;
      const int n_raw = seg0_raw ? max(0, min(seg0_nk, kb_hi) - kb_lo) : 0;
      // local k-block kb belongs to group (kb_run + kb) % GROUPS
      const int kb0 = ((grp - kb_run % GROUPS) + GROUPS) % GROUPS;
      if (n_raw > 0) {
        // raw-staged NF4 k-blocks of this group.  The group scales of the group's NEXT k-block
        // are loaded while this one decodes, so their L2 latency never sits between a
        // k-block's raw data arriving and its decode.
        const bool fwd = p.seg[0].B.kind == OP_NF4_K;
        ScaleRegs<BN> cur, nxt;
        if (kb0 < n_raw) load_scales<BN>(p, fwd, n0, kb_lo + kb0, gtid, nxt);
        for (int kb = kb0; kb < n_raw; kb += GROUPS) {
          const int kk = kb_lo + kb;
          cur = nxt;
          if (kb + GROUPS < n_raw) load_scales<BN>(p, fwd, n0, kk + GROUPS, gtid, nxt);
          const int gb = kb_run + kb, rb = raw_run + kb;
          const int st = gb % C::STAGES;
          const uint32_t ph = static_cast<uint32_t>(gb / C::STAGES) & 1u;
          uint8_t* As = base + st * C::STAGE_BYTES;
          uint8_t* Bs = As + C::A_BYTES;
          const int rs = rb % C::RAW_SLOTS;
          const uint32_t rph = static_cast<uint32_t>(rb / C::RAW_SLOTS) & 1u;
          const uint8_t* Rc = raw_base + rs * C::RAW_BYTES;
          const uint8_t* Rq = Rc + C::RAW_CODE_BYTES;
          mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, p.err);
          mbar_wait_bounded(&raw_full[rs], rph, abort_flag, p.err);
          if (fwd) {
            decode_fwd_raw<BN>(p.nf4, nf4_seg_of(p.nf4, n0), cb, seg_mean, n0, p.N, kk, Rc, Rq, Bs, gtid, cur.v);
          } else {
            const int k0 = kk * BK;
            decode_dx_raw<BN>(p.nf4, nf4_seg_of(p.nf4, k0), cb, seg_mean, n0, p.N, k0, ((n0 >> 6) >> 4) << 4, Rc, Rq,
                              Bs, gtid, cur.v);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&raw_empty[rs]);  // this warp's reads of the raw slot are done
          if (p.a_mode[0] == 0) load_tile<BM>(p.seg[0].A, p.nf4, lut, seg_mean, p.seg[0].K, m0, p.M, kk * BK, As, gtid);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[st]);
        }
      }
      int g = 0;
      for (int s = 0; s < p.nseg; ++s) {
        const GemmSeg& sg = p.seg[s];
        if (!seg_active(sg, n0, BN)) continue;
        const int nk = (sg.K + BK - 1) / BK;
        if (s == 0 && p.raw_tma) {  // handled above
          g += nk;
          continue;
        }
        // only this piece's k-blocks of the segment, and of those only this group's (walking
        // the whole K and skipping cost ~100 ns per k-block: 20 us on a 224-k-block GEMM)
        const int lo = g > kb_lo ? g : kb_lo;
        const int hi = g + nk < kb_hi ? g + nk : kb_hi;
        const int first = lo + ((grp - (kb_run + lo - kb_lo) % GROUPS) + GROUPS) % GROUPS;
        g += nk;
        for (int gk = first; gk < hi; gk += GROUPS) {
          const int kk = gk - (g - nk);
          const int gb = kb_run + (gk - kb_lo);
          const int st = gb % C::STAGES;
          const uint32_t ph = static_cast<uint32_t>(gb / C::STAGES) & 1u;
          uint8_t* As = base + st * C::STAGE_BYTES;
          uint8_t* Bs = As + C::A_BYTES;
          {
            mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, p.err);
            if (p.b_mode[s] == 0) load_tile<BN>(sg.B, p.nf4, lut, seg_mean, sg.K, n0, p.N, kk * BK, Bs, gtid);
          }
          if (p.a_mode[s] == 0) load_tile<BM>(sg.A, p.nf4, lut, seg_mean, sg.K, m0, p.M, kk * BK, As, gtid);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[st]);
        }
      }
      kb_run += kb_hi > kb_lo ? kb_hi - kb_lo : 0;
      raw_run += n_raw;
    }
  } else {
    const int q = warp - EPI_WARP0;  // TMEM lane quarter of this epilogue warp
    int kb_run = 0, raw_run = 0;
    int mma_st = 0;  // MMA issuer's stage and phase (run on across pieces)
    uint32_t mma_ph = 0;
    for (int pc = 0; pc < n_pieces; ++pc) {
      const Piece z = piece_at<BM, BN, SK>(p, pc);
      const int n0 = z.n0, m0 = z.m0, kb_lo = z.kb_lo, kb_hi = z.kb_hi;
      const bool seg0_raw = p.raw_tma && seg_active(p.seg[0], n0, BN);
      const int seg0_nk = seg0_raw ? (p.seg[0].K + BK - 1) / BK : 0;
      const int n_raw = seg0_raw ? max(0, min(seg0_nk, kb_hi) - kb_lo) : 0;
      if (warp == EPI_WARP0 + 1 && lane == 0) {
        // ---------------------------------------------- TMA issuer: operand tiles (A, bf16 B)
        int g = 0;
        for (int s = 0; s < p.nseg; ++s) {
          const GemmSeg& sg = p.seg[s];
          if (!seg_active(sg, n0, BN)) continue;
          const int nk = (sg.K + BK - 1) / BK;
          const bool raw = (s == 0) && p.raw_tma;
          const int lo = g > kb_lo ? g : kb_lo;
          const int hi = g + nk < kb_hi ? g + nk : kb_hi;
          g += nk;
          for (int gk = lo; gk < hi; ++gk) {
            const int kk = gk - (g - nk);
            const int gb = kb_run + (gk - kb_lo);
            const int st = gb % C::STAGES;
            const uint32_t ph = static_cast<uint32_t>(gb / C::STAGES) & 1u;
            mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, p.err);
            uint8_t* As = base + st * C::STAGE_BYTES;
            uint8_t* Bs = As + C::A_BYTES;
            const int am = p.a_mode[s], bm = raw ? 0 : p.b_mode[s];
            const uint32_t tx = (am ? C::A_BYTES : 0) + (bm ? C::B_BYTES : 0);
            if (tx) {
              mbar_arrive_expect_tx(&full[st], tx);
              const int k0 = kk * BK;
              if (am == 1) {
                tma_load_2d(As, &p.tmapA[s], k0, m0, &full[st]);
              } else if (am == 2) {
#pragma unroll
                for (int i = 0; i < BM / 64; ++i) tma_load_2d(As + i * 8192, &p.tmapA[s], m0 + 64 * i, k0, &full[st]);
              }
              if (bm == 1) {
                tma_load_2d(Bs, &p.tmapB[s], k0, n0 - p.b_row0[s], &full[st]);
              } else if (bm == 2) {
#pragma unroll
                for (int i = 0; i < BN / 64; ++i) tma_load_2d(Bs + i * 8192, &p.tmapB[s], n0 + 64 * i, k0, &full[st]);
              }
            } else {
              mbar_arrive(&full[st]);
            }
          }
        }
      }
      if (warp == EPI_WARP0 + 2 && lane == 0 && n_raw > 0) {
        // ---------------------------------------------- TMA issuer: raw NF4 codes / absmax
        const GemmSeg& sg = p.seg[0];
        for (int kb = 0; kb < n_raw; ++kb) {
          const int kk = kb_lo + kb;  // k-block index within segment 0
          const int rb = raw_run + kb;
          const int rs = rb % C::RAW_SLOTS;
          const uint32_t rph = static_cast<uint32_t>(rb / C::RAW_SLOTS) & 1u;
          mbar_wait_bounded(&raw_empty[rs], rph ^ 1u, abort_flag, p.err);
          uint8_t* Rc = raw_base + rs * C::RAW_BYTES;
          uint8_t* Rq = Rc + C::RAW_CODE_BYTES;
          if (sg.B.kind == OP_NF4_K) {
            const int si = nf4_seg_of(p.nf4, n0);
            const int y = n0 - p.nf4.seg[si].row_begin;
            mbar_arrive_expect_tx(&raw_full[rs], BN * 32 + BN * 16);
            tma_load_2d(Rc, &p.tmapCodes[si], kk * (BK / 2), y, &raw_full[rs]);
            tma_load_2d(Rq, &p.tmapQ8[si], (kk >> 4) << 4, y, &raw_full[rs]);
          } else {
            const int k0 = kk * BK;
            const int si = nf4_seg_of(p.nf4, k0);
            const int y = k0 - p.nf4.seg[si].row_begin;
            mbar_arrive_expect_tx(&raw_full[rs], 64 * (BN / 2) + 64 * 16);
            tma_load_2d(Rc, &p.tmapCodes[si], n0 / 2, y, &raw_full[rs]);
            tma_load_2d(Rq, &p.tmapQ8[si], ((n0 >> 6) >> 4) << 4, y, &raw_full[rs]);
          }
        }
      }
      if (warp == EPI_WARP0 && lane == 0) {
        // ---------------------------------------------- MMA issuer
        // One thread; its per-k-block overhead sits between the tensor core's instructions,
        // so the loop keeps it small: the stage index and phase advance by increments,
        // operand descriptors by plain adds (the start-address field is the byte address / 16
        // and stays inside its 14 bits in shared memory), and the stage's full barrier is
        // probed with test_wait before the blocking wait.  A piece after the first waits until
        // the epilogue has read the previous piece's accumulator out of TMEM.
        if (pc > 0) mbar_wait_bounded(tmem_empty, static_cast<uint32_t>(pc - 1) & 1u, abort_flag, p.err);
        tc_fence_after();
        const uint32_t smem0 = smem_u32(base);
        int g = 0, kb = 0;
        for (int s = 0; s < p.nseg; ++s) {
          const GemmSeg& sg = p.seg[s];
          if (!seg_active(sg, n0, BN)) continue;
          const int nk = (sg.K + BK - 1) / BK;
          const int lo = g > kb_lo ? g : kb_lo;
          const int hi = g + nk < kb_hi ? g + nk : kb_hi;
          g += nk;
          if (lo >= hi) continue;
          const bool b_mn = ((s == 0) && p.raw_tma && sg.B.kind == OP_NF4_MN) || p.b_mode[s] == 2;
          const bool a_mn = p.a_mode[s] == 2;
          const uint32_t idesc = idesc_bf16_f32<BN>(a_mn, b_mn);
          const uint64_t a0 = a_mn ? sw128_mnmajor_desc(smem0) : sw128_kmajor_desc(smem0);
          const uint64_t b0 = b_mn ? sw128_mnmajor_desc(smem0 + C::A_BYTES) : sw128_kmajor_desc(smem0 + C::A_BYTES);
          const uint64_t aj = a_mn ? (2048u >> 4) : (32u >> 4);  // one K = 16 step, in 16-byte units
          const uint64_t bj = b_mn ? (2048u >> 4) : (32u >> 4);
          for (int it = lo; it < hi; ++it) {
            if (!mbar_test_wait(&full[mma_st], mma_ph)) mbar_wait_bounded(&full[mma_st], mma_ph, abort_flag, p.err);
            tc_fence_after();
            const uint64_t so = static_cast<uint64_t>(mma_st) * (C::STAGE_BYTES >> 4);
#pragma unroll
            for (int j = 0; j < BK / 16; ++j) {
              const uint64_t bd = b0 + so + j * bj;
#pragma unroll
              for (int h = 0; h < MT; ++h) {  // the 128-row halves share the B tile (one dequant)
                const uint64_t ad = a0 + so + h * ((UM * 128) >> 4) + j * aj;
                tc_mma_f16(tmem + h * BN, ad, bd, idesc, (kb > 0 || j > 0) ? 1u : 0u);
              }
            }
            tc_commit(&empty[mma_st]);
            ++kb;
            if (++mma_st == C::STAGES) {
              mma_st = 0;
              mma_ph ^= 1u;
            }
          }
        }
        tc_commit(done);
      }
      __syncwarp();
      // ---------------------------------------------- epilogue (warps 12..15 = TMEM lane quarters 0..3)
      mbar_wait_bounded(done, static_cast<uint32_t>(pc) & 1u, abort_flag, p.err);
      tc_fence_after();
      const bool any_k = kb_hi > kb_lo;
      const bool sk_part = SK && z.partial;
      float* slot = sk_part ? p.workspace + static_cast<long long>(sk_slot(blockIdx.x, pc)) * (BM * BN) : nullptr;
      const bool rope_tile = p.rope_cols > 0 && n0 < p.rope_cols && !z.partial && any_k;
      if (rope_tile) {
        // head pairs (i, i + d/2) are both in this tile (tiles never straddle a head: see gemm_plan)
        const int half = p.rope_d >> 1;
#pragma unroll 1
        for (int h = 0; h < MT; ++h)
#pragma unroll 1
          for (int hb = 0; hb < BN; hb += p.rope_d)
#pragma unroll 1
            for (int i0 = 0; i0 < half; i0 += 16) {
              const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(h * BN + hb + i0);
              uint32_t a[16], b[16];
              tmem_ld16(tq, a);
              tmem_ld16(tq + static_cast<uint32_t>(half), b);
              tmem_ld_wait();
              const int row = m0 + h * UM + q * 32 + lane;
              if (row < p.M) rope_store16(p, row, n0 + hb, i0, a, b);
            }
      }
#pragma unroll 1
      for (int hc = 0; hc < (rope_tile ? 0 : MT * BN); hc += 16) {
        const int h = hc / BN, cc = hc % BN;
        const int rl = h * UM + q * 32 + lane;  // row within the tile
        const int row = m0 + rl;
        uint32_t r[16];
        tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(hc), r);
        tmem_ld_wait();
        const int col0 = n0 + cc;
        if (row >= p.M || col0 >= p.N) continue;
        if (z.partial) {
          float4* o = sk_part ? reinterpret_cast<float4*>(slot + rl * BN + cc)
                              : reinterpret_cast<float4*>(p.workspace +
                                                          (static_cast<long long>(blockIdx.z) * p.M + row) * p.N + col0);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            if (col0 + g * 4 >= p.N) break;
            o[g] = any_k ? make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                                       __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3]))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        } else {
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = any_k ? p.alpha * __uint_as_float(r[j]) : 0.f;
          epilogue_store<16>(p, row, col0, v);
        }
      }
      // the accumulator is out of TMEM: the next piece's MMAs may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_empty);
      kb_run += kb_hi > kb_lo ? kb_hi - kb_lo : 0;
      raw_run += n_raw;
    }
  }

  tc_fence_before();
  if (splits > 1 && p.fused_reduce) __threadfence();  // this CTA's partial tile, visible before its ticket
  __syncthreads();
  if (warp == EPI_WARP0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (splits > 1 && p.fused_reduce) {
    // The last split of this tile to finish sums every partial in split order (the same
    // arithmetic, in the same order, as the separate reduction kernel) with all 512 threads:
    // one (row, 8-column group) per thread at a time, every split's loads issued together.
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    if (threadIdx.x == 0) {
      const int tile = blockIdx.y * gridDim.x + blockIdx.x;
      const int old = atomicAdd(&p.tile_counters[tile], 1);
      const int last = (old == splits - 1) ? 1 : 0;
      if (last) p.tile_counters[tile] = 0;  // every split has counted: ready for the next launch
      *last_flag = last;
    }
    __syncthreads();
    if (*last_flag) {
      __threadfence();
      constexpr int G8 = BN / 8;
#pragma unroll 1
      for (int it = threadIdx.x; it < BM * G8; it += GEMM_THREADS) {
        const int row = m0 + it / G8, col0 = n0 + (it % G8) * 8;
        if (row >= p.M || col0 >= p.N) continue;
        float4 a[4][2];
#pragma unroll
        for (int sp = 0; sp < 4; ++sp) {
          if (sp >= splits) break;
          const float4* src =
              reinterpret_cast<const float4*>(p.workspace + (static_cast<long long>(sp) * p.M + row) * p.N + col0);
          a[sp][0] = __ldcg(src);
          a[sp][1] = __ldcg(src + 1);
        }
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int sp = 0; sp < 4; ++sp) {
          if (sp >= splits) break;
          v[0] += a[sp][0].x; v[1] += a[sp][0].y; v[2] += a[sp][0].z; v[3] += a[sp][0].w;
          v[4] += a[sp][1].x; v[5] += a[sp][1].y; v[6] += a[sp][1].z; v[7] += a[sp][1].w;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] *= p.alpha;
        epilogue_store<8>(p, row, col0, v);
      }
    }
  }
}

// ---------------------------------------------------------------- the TMEM-A forward kernel
// NF4 forward GEMMs with enough output tiles (y = x W^T (+ LoRA K-blocks) (+ residual), RoPE on
// the q | k columns): the tile is transposed, D^T[w, t] = W[w, :] . x[t, :], 128 weight rows
// (TMEM lanes) x 256 tokens.
// The producers put the dequantised weight tile straight into tensor memory (tcgen05.st, one
// weight row per thread) and tcgen05.mma reads it there as its A operand; only the activation
// tile (TMA) and the raw NF4 bytes pass through shared memory.  Against the shared-memory form
// (activations and decoded weights both staged in shared memory and both read by every MMA)
// this moves ~76 KB of shared memory per 4.2 MFLOP k-block instead of ~124 KB.  LoRA segments
// are further K-blocks: the producers copy the LoRA-B rows of the tile (bf16, zero outside the
// segment's row window) into tensor memory and the u tile comes by TMA.  The epilogue's
// per-(token, column) inputs, the residual block or the tile's 256 positions' cos / sin rows,
// come by TMA as further entries of the activation ring, into the stages the last k-blocks
// free first, and are read from shared memory: in the transposed tile a thread walks tokens,
// and fetching those values from global memory one token at a time made the q|k|v launch 182 us
// against 58 in the 8B step.
struct TsCfg {
  static constexpr int BW = 128;  // weight rows (output columns) per CTA
  static constexpr int BT = 256;  // tokens (output rows) per CTA: the MMA's N
  static constexpr int STAGES = 5;
  static constexpr int RAW_SLOTS = 6;
  static constexpr int X_BYTES = BT * 128;
  static constexpr int RAW_CODE_BYTES = BW * 32, RAW_Q8_BYTES = BW * 16;
  static constexpr int RAW_BYTES = RAW_CODE_BYTES + RAW_Q8_BYTES;
  static constexpr int CTRL_BYTES = 512;
  static constexpr int SMEM_BYTES = 1024 + STAGES * X_BYTES + RAW_SLOTS * RAW_BYTES + CTRL_BYTES;
  static constexpr int ACC_COL = 0, W_COL = BT, TMEM_COLS = 512;
};
static_assert(TsCfg::W_COL + TsCfg::STAGES * 32 <= TsCfg::TMEM_COLS, "TMEM budget");
static_assert(TsCfg::RAW_SLOTS >= TsCfg::STAGES && TsCfg::STAGES >= GROUPS, "ring invariants");
static_assert(TsCfg::SMEM_BYTES <= SMEM_LIMIT, "shared memory");

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__global__ void __launch_bounds__(GEMM_THREADS, 1) gemm_ts_kernel(const __grid_constant__ GemmParams p) {
  using C = TsCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* raw_base = base + C::STAGES * C::X_BYTES;
  uint8_t* ctrl = raw_base + C::RAW_SLOTS * C::RAW_BYTES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl + 4);
  float* seg_mean = reinterpret_cast<float*>(ctrl + 16);  // up to 3 NF4 tensors
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl + 64);
  uint64_t* empty = full + C::STAGES;
  uint64_t* raw_full = empty + C::STAGES;
  uint64_t* raw_empty = raw_full + C::RAW_SLOTS;
  uint64_t* done = raw_empty + C::RAW_SLOTS;
  uint64_t* res_full = done + 1;
  static_assert(64 + 8 * (2 * C::STAGES + 2 * C::RAW_SLOTS + 2) <= C::CTRL_BYTES, "control block overflow");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * C::BW;  // first weight row = output column
  const int m0 = blockIdx.y * C::BT;  // first token = output row
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], GROUP_THREADS / 32 + 1);  // 4 producer warps + the activation TMA issuer
      mbar_init(&empty[s], 1);
    }
    for (int r = 0; r < C::RAW_SLOTS; ++r) {
      mbar_init(&raw_full[r], 1);
      mbar_init(&raw_empty[r], GROUP_THREADS / 32);
    }
    mbar_init(done, 1);
    mbar_init(res_full, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (threadIdx.x >= 32 && threadIdx.x < 32 + p.nf4.nseg) seg_mean[threadIdx.x - 32] = *p.nf4.seg[threadIdx.x - 32].mean;
  if (warp == EPI_WARP0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // segment 0: the NF4 weight (raw-staged); then the active LoRA segments, one after another
  const int nk0 = p.seg[0].K / BK;  // a multiple of 16 k-blocks (raw staging needs it)

  if (warp < PRODUCER_WARPS) {
    // ---------------------------------------------- producers: weight row r of the tile = TMEM lane r
    const int grp = warp >> 2, r = threadIdx.x & (GROUP_THREADS - 1);
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float(&cb)[16] = p.lut;
    const int w = n0 + r;
    const int si = nf4_seg_of(p.nf4, n0);
    const NF4Seg& ns = p.nf4.seg[si];
    const long long cpr = p.nf4.cols >> 6;
    int kb = 0;
    for (int s = 0; s < p.nseg; ++s) {
      const GemmSeg& sg = p.seg[s];
      if (!seg_active(sg, n0, C::BW)) continue;
      const int nk = (sg.K + BK - 1) / BK;
      const int first = kb + ((grp - kb % GROUPS) + GROUPS) % GROUPS;
      for (int g = first; g < kb + nk; g += GROUPS) {
        const int kk = g - kb;  // k-block within the segment
        const int st = g % C::STAGES;
        const uint32_t ph = static_cast<uint32_t>(g / C::STAGES) & 1u;
        uint32_t o[32];
        if (s == 0) {
          const int rs = g % C::RAW_SLOTS;
          const uint32_t rph = static_cast<uint32_t>(g / C::RAW_SLOTS) & 1u;
          const float s2 = (w < p.N) ? __ldg(ns.scales + ((static_cast<long long>(w - ns.row_begin) * cpr + kk) >> 8))
                                     : 0.f;
          mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, p.err);
          mbar_wait_bounded(&raw_full[rs], rph, abort_flag, p.err);
          const uint32_t rc = smem_u32(raw_base + rs * C::RAW_BYTES) + r * 32;
          const uint4 w0 = lds128(rc), w1 = lds128(rc + 16);
          const int q8 = lds_s8(smem_u32(raw_base + rs * C::RAW_BYTES + C::RAW_CODE_BYTES) + r * 16 + (kk & 15));
          __syncwarp();
          if (lane == 0) mbar_arrive(&raw_empty[rs]);  // this warp's reads of the raw slot are done
          const float mh = __fadd_rn(__fmul_rn(static_cast<float>(q8), s2), seg_mean[si]);
          const BlockLut t = block_lut(cb, mh);
          const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
          for (int kc = 0; kc < 8; ++kc) {
            const uint4 v = decode_word_lut(words[kc], t);
            o[4 * kc] = v.x;
            o[4 * kc + 1] = v.y;
            o[4 * kc + 2] = v.z;
            o[4 * kc + 3] = v.w;
          }
          if (w >= p.N) {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
        } else {
          // LoRA-B row w (bf16, K-major): columns kk*64 .. +64 of K, zero outside the row window
          const bool in = w < p.N && w >= sg.B.row_lo && w < sg.B.row_hi;
          const int k0 = kk * BK;
          const uint16_t* src = static_cast<const uint16_t*>(sg.B.ptr) + static_cast<long long>(w) * sg.B.ld + k0;
          uint4 v[8];
#pragma unroll
          for (int c = 0; c < 8; ++c)
            v[c] = (in && k0 + c * 8 < sg.K) ? *reinterpret_cast<const uint4*>(src + c * 8) : make_uint4(0, 0, 0, 0);
          mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, p.err);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            o[4 * c] = v[c].x;
            o[4 * c + 1] = v[c].y;
            o[4 * c + 2] = v[c].z;
            o[4 * c + 3] = v[c].w;
          }
        }
        tmem_st32(tmem + lane_base + C::W_COL + st * 32, o);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[st]);
      }
      kb += nk;
    }
  } else {
    const int q = warp - EPI_WARP0;  // TMEM lane quarter of this epilogue warp
    if (warp == EPI_WARP0 + 1 && lane == 0) {
      // ---------------------------------------------- TMA issuer: the token tiles (x, then u)
      int kb = 0;
      for (int s = 0; s < p.nseg; ++s) {
        const GemmSeg& sg = p.seg[s];
        if (!seg_active(sg, n0, C::BW)) continue;
        const int nk = (sg.K + BK - 1) / BK;
        for (int kk = 0; kk < nk; ++kk, ++kb) {
          const int st = kb % C::STAGES;
          const uint32_t ph = static_cast<uint32_t>(kb / C::STAGES) & 1u;
          mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, p.err);
          mbar_arrive_expect_tx(&full[st], C::X_BYTES);
          tma_load_2d(base + st * C::X_BYTES, &p.tmapA[s], kk * BK, m0, &full[st]);
        }
      }
      if (p.residual) {
        // residual rows [m0, m0 + 128) and [m0 + 128, m0 + 256) into the stages that ring
        // entries kb and kb + 1 would use (free once the MMAs five entries back retire)
        mbar_arrive_expect_tx(res_full, 2 * 128 * C::BW * 2);
        for (int h = 0; h < 2; ++h) {
          const int g = kb + h, st = g % C::STAGES;
          const uint32_t ph = static_cast<uint32_t>(g / C::STAGES) & 1u;
          mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, p.err);
          tma_load_2d(base + st * C::X_BYTES, &p.tmapB[0], n0, m0 + 128 * h, res_full);
        }
      } else if (p.rope_cols > 0 && n0 < p.rope_cols) {
        // cos rows of positions [pos0, pos0 + 128), [pos0 + 128, +256), then the sin rows, as
        // ring entries kb .. kb + 3 (the tile's tokens have consecutive positions)
        const int pos0 = m0 % p.rope_S;
        mbar_arrive_expect_tx(res_full, 4 * 128 * 64 * 4);
        for (int e = 0; e < 4; ++e) {
          const int g = kb + e, st = g % C::STAGES;
          const uint32_t ph = static_cast<uint32_t>(g / C::STAGES) & 1u;
          mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, p.err);
          tma_load_2d(base + st * C::X_BYTES, &p.tmapB[1 + (e >> 1)], 0, pos0 + 128 * (e & 1), res_full);
        }
      }
    }
    if (warp == EPI_WARP0 + 2 && lane == 0) {
      // ---------------------------------------------- TMA issuer: raw NF4 codes / absmax
      const int si = nf4_seg_of(p.nf4, n0);
      const int y = n0 - p.nf4.seg[si].row_begin;
      for (int kb = 0; kb < nk0; ++kb) {
        const int rs = kb % C::RAW_SLOTS;
        const uint32_t rph = static_cast<uint32_t>(kb / C::RAW_SLOTS) & 1u;
        mbar_wait_bounded(&raw_empty[rs], rph ^ 1u, abort_flag, p.err);
        uint8_t* Rc = raw_base + rs * C::RAW_BYTES;
        mbar_arrive_expect_tx(&raw_full[rs], C::RAW_BYTES);
        tma_load_2d(Rc, &p.tmapCodes[si], kb * (BK / 2), y, &raw_full[rs]);
        tma_load_2d(Rc + C::RAW_CODE_BYTES, &p.tmapQ8[si], (kb >> 4) << 4, y, &raw_full[rs]);
      }
    }
    if (warp == EPI_WARP0 && lane == 0) {
      // ---------------------------------------------- MMA issuer: A (weights) from TMEM
      const uint32_t idesc = idesc_bf16(C::BW, C::BT, false, false);
      const uint32_t x0 = smem_u32(base);
      int st = 0, kb = 0;
      uint32_t ph = 0;
      for (int s = 0; s < p.nseg; ++s) {
        const GemmSeg& sg = p.seg[s];
        if (!seg_active(sg, n0, C::BW)) continue;
        const int nk = (sg.K + BK - 1) / BK;
        for (int kk = 0; kk < nk; ++kk, ++kb) {
          if (!mbar_test_wait(&full[st], ph)) mbar_wait_bounded(&full[st], ph, abort_flag, p.err);
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < BK / 16; ++j)
            tc_mma_f16_ts(tmem + C::ACC_COL, tmem + C::W_COL + st * 32 + j * 8,
                          sw128_kmajor_desc(x0 + st * C::X_BYTES + j * 32), idesc, (kb > 0 || j > 0) ? 1u : 0u);
          tc_commit(&empty[st]);
          if (++st == C::STAGES) {
            st = 0;
            ph ^= 1u;
          }
        }
      }
      tc_commit(done);
    }
    __syncwarp();
    // ------------------------------------------------ epilogue: thread = output column w
    mbar_wait_bounded(done, 0u, abort_flag, p.err);
    tc_fence_after();
    const int w = n0 + q * 32 + lane;
    uint16_t* out = static_cast<uint16_t*>(p.out);
    int nkb_all = 0;
    for (int s = 0; s < p.nseg; ++s)
      if (seg_active(p.seg[s], n0, C::BW)) nkb_all += (p.seg[s].K + BK - 1) / BK;
    const bool rope_tile = !p.residual && p.rope_cols > 0 && n0 < p.rope_cols;
    if (p.residual || rope_tile) mbar_wait_bounded(res_full, 0u, abort_flag, p.err);
    const uint8_t* rs0 = base + (nkb_all % C::STAGES) * C::X_BYTES;
    const uint8_t* rs1 = base + ((nkb_all + 1) % C::STAGES) * C::X_BYTES;
    const float* cos0 = reinterpret_cast<const float*>(rs0);
    const float* cos1 = reinterpret_cast<const float*>(rs1);
    const float* sin0 = reinterpret_cast<const float*>(base + ((nkb_all + 2) % C::STAGES) * C::X_BYTES);
    const float* sin1 = reinterpret_cast<const float*>(base + ((nkb_all + 3) % C::STAGES) * C::X_BYTES);
    // the pair exchange in the stage of the last k-block (ring entry nkb_all - 1 = nkb_all + 4)
    float* xch = reinterpret_cast<float*>(base + ((nkb_all + 4) % C::STAGES) * C::X_BYTES);
    const int dr = q * 32 + lane, pdr = dr ^ 64, ci = dr & 63;
    const bool first = dr < 64;
#pragma unroll 1
    for (int tc = 0; tc < C::BT; tc += 16) {
      uint32_t acc[16];
      tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + C::ACC_COL + tc, acc);
      tmem_ld_wait();
      float v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = p.alpha * __uint_as_float(acc[j]);
      if (p.residual) {
        const uint8_t* rb = (tc < 128 ? rs0 : rs1) + (tc & 127) * (C::BW * 2) + (q * 32 + lane) * 2;
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] += bf16_to_f32(*reinterpret_cast<const uint16_t*>(rb + j * C::BW * 2));
      }
      if (rope_tile) {
        // rows dr and dr ^ 64 of the tile are the pair (i, i + 64) of one head
#pragma unroll
        for (int j = 0; j < 16; ++j) xch[dr * 17 + j] = v[j];
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const float* ct = (tc < 128 ? cos0 : cos1) + (tc & 127) * 64 + ci;
        const float* stb = (tc < 128 ? sin0 : sin1) + (tc & 127) * 64 + ci;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float other = xch[pdr * 17 + j];
          const float c = ct[j * 64], sn = stb[j * 64];
          const float x1 = first ? v[j] : other, x2 = first ? other : v[j];
          v[j] = first ? x1 * c - x2 * sn : x2 * c + x1 * sn;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
      if (w < p.N) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = m0 + tc + j;
          if (t < p.M) {
            const __nv_bfloat16 b = __float2bfloat16_rn(v[j]);
            out[static_cast<long long>(t) * p.ldo + w] = *reinterpret_cast<const uint16_t*>(&b);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == EPI_WARP0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Sum of the split-K partial tiles in split order, then the normal epilogue (the wide form
// for many splits: one thread per 8 outputs instead of one CTA per tile, 128-thread blocks so
// that the few thousand threads of a LoRA-sized output spread over more SMs).
__global__ void splitk_reduce_kernel(const __grid_constant__ GemmParams p) {
  const long long n8 = p.N / 8;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(p.M) * n8) return;
  const int row = static_cast<int>(idx / n8), col = static_cast<int>(idx % n8) * 8;
  float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  // eight splits' loads in flight at a time, added in split order
#pragma unroll 1
  for (int s0 = 0; s0 < p.splits; s0 += 8) {
    float4 a[8][2];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (s0 + u >= p.splits) break;
      const float4* src =
          reinterpret_cast<const float4*>(p.workspace + (static_cast<long long>(s0 + u) * p.M + row) * p.N + col);
      a[u][0] = __ldcg(src);
      a[u][1] = __ldcg(src + 1);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (s0 + u >= p.splits) break;
      v[0] += a[u][0].x; v[1] += a[u][0].y; v[2] += a[u][0].z; v[3] += a[u][0].w;
      v[4] += a[u][1].x; v[5] += a[u][1].y; v[6] += a[u][1].z; v[7] += a[u][1].w;
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] *= p.alpha;
  epilogue_store<8>(p, row, col, v);
}

// Stream-K: every tile cut between CTAs summed share by share in k order (CTA order, the order
// a single CTA's k loop would have added them) and written through the normal epilogue, one
// thread per (row, 8 columns), all cut tiles at once.  A tile one CTA computed whole was
// written by that CTA.  Block x looks at the boundary between CTAs x and x + 1: the tile it
// falls in is cut (unless the boundary is a tile boundary) and is summed by the blocks of its
// first such boundary; blocks y cover the tile's rows.  A separate launch: summed at the end of
// the CTA that completed a tile, the shares' loads (up to 4 x 128 KB, one SM) added a ~20 us
// tail to the long GEMMs.
template <int BM, int BN>
__global__ void sk_fixup_kernel(const __grid_constant__ GemmParams p) {
  const int c = blockIdx.x + 1;  // boundary between CTAs c - 1 and c
  const long long xb = sk_bound(p.sk_tiles, p.sk_nkt, p.sk_ctas, c);
  if (xb % p.sk_nkt == 0) return;  // not inside a tile
  const int t = static_cast<int>(xb / p.sk_nkt);
  const long long xp = sk_bound(p.sk_tiles, p.sk_nkt, p.sk_ctas, c - 1);
  if (c > 1 && xp / p.sk_nkt == t && xp % p.sk_nkt != 0) return;  // an earlier boundary cut this tile
  const long long x0 = static_cast<long long>(t) * p.sk_nkt;
  const int cf = sk_owner(p.sk_tiles, p.sk_nkt, p.sk_ctas, x0);
  const int nsh = sk_owner(p.sk_tiles, p.sk_nkt, p.sk_ctas, x0 + p.sk_nkt - 1) - cf + 1;
  if (nsh < 2) return;
  if (nsh > 4) {  // the planner cuts a tile into at most 4 shares
    if (threadIdx.x == 0 && blockIdx.y == 0) set_dev_error(p.err, DEVERR_BOUNDS);
    return;
  }
  constexpr int G8 = BN / 8;
  const int it = blockIdx.y * blockDim.x + threadIdx.x;
  if (it >= BM * G8) return;
  const int m0 = (t % p.sk_tiles_m) * BM, n0 = (t / p.sk_tiles_m) * BN;
  const int rl = it / G8, cl8 = (it % G8) * 8;
  const int row = m0 + rl, col0 = n0 + cl8;
  if (row >= p.M || col0 >= p.N) return;
  // share 0 sits in CTA cf's last-piece slot when the tile began inside its range, the others
  // in their CTAs' first-piece slots
  int c0, sl0;
  sk_share(p.sk_tiles, p.sk_nkt, p.sk_ctas, t, 0, &c0, &sl0);
  float4 a[4][2];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (k >= nsh) break;
    const long long slot = k == 0 ? sl0 : 2LL * (cf + k);
    const float4* src = reinterpret_cast<const float4*>(p.workspace + slot * (BM * BN) + rl * BN + cl8);
    a[k][0] = __ldcg(src);
    a[k][1] = __ldcg(src + 1);
  }
  float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (k >= nsh) break;
    v[0] += a[k][0].x; v[1] += a[k][0].y; v[2] += a[k][0].z; v[3] += a[k][0].w;
    v[4] += a[k][1].x; v[5] += a[k][1].y; v[6] += a[k][1].z; v[7] += a[k][1].w;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] *= p.alpha;
  epilogue_store<8>(p, row, col0, v);
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// Encoded descriptors are cached by their arguments: the same activation and weight buffers
// recur every layer and every step, and encoding costs host time on every GEMM launch.
struct MapKey {
  const void* ptr;
  unsigned long long d0, d1, stride, d2, stride2;  // d2 = 0: a 2D map
  unsigned b0, b1, b2, pad;
  int dtype, swizzle;
  bool operator==(const MapKey& o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    const unsigned long long* w = reinterpret_cast<const unsigned long long*>(&k);
    unsigned long long h = 1469598103934665603ull;
    for (size_t i = 0; i < sizeof(MapKey) / 8; ++i) h = (h ^ w[i]) * 1099511628211ull;
    return static_cast<size_t>(h);
  }
};
bool encode_cached(CUtensorMap* map, const void* ptr, CUtensorMapDataType dtype, unsigned long long d0,
                   unsigned long long d1, unsigned long long stride_bytes, unsigned b0, unsigned b1,
                   CUtensorMapSwizzle swz, unsigned long long d2 = 0, unsigned long long stride2 = 0,
                   unsigned b2 = 1) {
  static std::mutex mu;
  static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
  MapKey key;
  std::memset(&key, 0, sizeof(key));
  key.ptr = ptr;
  key.d0 = d0;
  key.d1 = d1;
  key.stride = stride_bytes;
  key.b0 = b0;
  key.b1 = b1;
  key.d2 = d2;
  key.stride2 = stride2;
  key.b2 = d2 ? b2 : 0;
  key.dtype = static_cast<int>(dtype);
  key.swizzle = static_cast<int>(swz);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *map = it->second;
      return true;
    }
  }
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint32_t rank = d2 ? 3 : 2;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride_bytes, stride2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t es[3] = {1, 1, 1};
  if (fn(map, dtype, rank, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() > 8192) cache.clear();
  cache.emplace(key, *map);
  return true;
}

// TMA descriptor for a K-major bf16 operand: dims (K, rows), row stride ld elements, 64 x
// box_rows box, 128-byte swizzle (the layout the MMA descriptors expect), zero fill.
bool encode_kmajor_bf16(CUtensorMap* map, const void* ptr, int K, int rows, long long ld, int box_rows) {
  if (K <= 0 || rows <= 0) return false;
  return encode_cached(map, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<unsigned long long>(K),
                       static_cast<unsigned long long>(rows), static_cast<unsigned long long>(ld) * 2, BK,
                       static_cast<unsigned>(box_rows), CU_TENSOR_MAP_SWIZZLE_128B);
}

// TMA descriptor for an MN-major bf16 operand (element (r, k) at ptr[k*ld + r]): dims (rows, K),
// 64 x 64 boxes with 128-byte swizzle = one MN-major atom column of a 64-deep K block.
bool encode_mnmajor_bf16(CUtensorMap* map, const void* ptr, int rows, int K, long long ld) {
  if (K <= 0 || rows <= 0) return false;
  return encode_cached(map, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<unsigned long long>(rows),
                       static_cast<unsigned long long>(K), static_cast<unsigned long long>(ld) * 2, 64, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B);
}

// TMA descriptor for a 2D uint8 array (raw NF4 codes or q8 absmax), no swizzle, zero fill.
bool encode_u8_2d(CUtensorMap* map, const void* ptr, unsigned long long w, unsigned long long h,
                  unsigned long long stride, unsigned box_w, unsigned box_h) {
  return encode_cached(map, ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, h, stride, box_w, box_h,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Raw TMA staging of the NF4 operand: rows of 1024-column multiples (so the q8 absmax rows are
// 16-byte multiples) and tiles that never straddle two stacked tensors.
bool raw_tma_allowed() {
  static const bool allowed = [] {
    const char* e = std::getenv("SOUP_GEMM_RAW_TMA");
    return !(e && e[0] == '0');
  }();
  return allowed;
}

// SOUP_GEMM_TMA_OPERANDS=0 keeps every operand except K-major A on the producer-warp path.
bool tma_operands_allowed() {
  static const bool allowed = [] {
    const char* e = std::getenv("SOUP_GEMM_TMA_OPERANDS");
    return !(e && e[0] == '0');
  }();
  return allowed;
}

bool setup_raw_tma(GemmParams& p, int BN) {
  if (!raw_tma_allowed()) return false;
  const GemmSeg& s0 = p.seg[0];
  if (s0.K <= 0 || (s0.B.kind != OP_NF4_K && s0.B.kind != OP_NF4_MN)) return false;
  const NF4Group& g = p.nf4;
  if (g.cols % 1024 != 0 || g.nseg < 1) return false;
  if (s0.B.kind == OP_NF4_K) {
    for (int i = 1; i < g.nseg; ++i)
      if (g.seg[i].row_begin % BN != 0) return false;
  } else {
    if (p.N != g.cols) return false;
    for (int i = 1; i < g.nseg; ++i)
      if (g.seg[i].row_begin % 64 != 0) return false;
  }
  const unsigned long long cb = static_cast<unsigned long long>(g.cols) / 2, qb = static_cast<unsigned long long>(g.cols) / 64;
  for (int i = 0; i < g.nseg; ++i) {
    const unsigned long long rows = static_cast<unsigned long long>(g.seg[i].rows);
    const bool ok = (s0.B.kind == OP_NF4_K)
                        ? (encode_u8_2d(&p.tmapCodes[i], g.seg[i].codes, cb, rows, cb, 32, BN) &&
                           encode_u8_2d(&p.tmapQ8[i], g.seg[i].q8, qb, rows, qb, 16, BN))
                        : (encode_u8_2d(&p.tmapCodes[i], g.seg[i].codes, cb, rows, cb, BN / 2, 64) &&
                           encode_u8_2d(&p.tmapQ8[i], g.seg[i].q8, qb, rows, qb, 16, 64));
    if (!ok) return false;
  }
  return true;
}

template <int MT, int BN, bool SK = false>
cudaError_t launch_tile(const GemmParams& p, cudaStream_t st) {
  using C = GemmCfg<MT, BN>;
  static_assert(C::STAGES >= 2, "tile too large for shared memory");
  // Producer group g fills the k-blocks g, g + GROUPS, ...; when it waits for a stage to free,
  // the stage's barrier must be at most one phase behind the one it needs, which holds when its
  // own previous k-block (GROUPS back) already required the MMAs of that stage's previous use:
  // STAGES >= GROUPS.  (With fewer stages a group can pass a parity check two phases early and
  // arrive on a barrier that is still collecting the previous k-block.)
  static_assert(C::STAGES >= GROUPS, "each producer group needs a stage of its own in flight");
  static_assert(C::RAW_SLOTS >= C::STAGES, "a raw slot's parity wait needs a slot per operand stage");
  static std::atomic<int> attr_done{0};
  if (!attr_done.load()) {
    cudaError_t e =
        cudaFuncSetAttribute(gemm_tc_kernel<MT, BN, SK>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done.store(1);
  }
  const dim3 grid = p.sk_ctas > 0 ? dim3(p.sk_ctas, 1, 1)
                                  : dim3((p.N + BN - 1) / BN, (p.M + C::BM - 1) / C::BM, p.splits > 1 ? p.splits : 1);
  gemm_tc_kernel<MT, BN, SK><<<grid, GEMM_THREADS, C::SMEM_BYTES, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (SK) {
    // the cut tiles' shares, summed by a wide second kernel
    constexpr int ITEMS = C::BM * BN / 8;
    if (p.sk_ctas > 1)
      sk_fixup_kernel<C::BM, BN><<<dim3(static_cast<unsigned>(p.sk_ctas - 1), (ITEMS + 511) / 512), 512, 0, st>>>(p);
    ++g_kernel_launches;
    return cudaGetLastError();
  }
  if (p.splits <= 1 || p.fused_reduce) return e;
  const long long work = static_cast<long long>(p.M) * (p.N / 8);
  splitk_reduce_kernel<<<static_cast<unsigned>((work + 127) / 128), 128, 0, st>>>(p);
  ++g_kernel_launches;
  return cudaGetLastError();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The TMEM-A forward kernel (gemm_ts_kernel) serves forward NF4 GEMMs without accumulation or
// fp32 / transposed output, whose LoRA segments are plain bf16 operands, when they have at least
// TS_MIN_TILES 128 x 256 output tiles (fewer tiles leave SMs idle: the shared-memory kernel's
// 128-column tiles, split-K or stream-K serve those).  A residual is a bf16 block of the output's
// shape; RoPE needs 128-column heads, whole 256-token tiles of consecutive positions and no
// shared-prefix pair layout.  SOUP_GEMM_TS=0 turns it off (read per launch).
constexpr int TS_MIN_TILES = 96;
bool ts_enabled() {
  const char* e = std::getenv("SOUP_GEMM_TS");
  return !(e && e[0] == '0');
}
bool ts_applicable(const GemmParams& p) {
  if (!ts_enabled() || !tma_operands_allowed() || !raw_tma_allowed()) return false;
  if (p.nseg < 1 || p.seg[0].K <= 0 || p.seg[0].B.kind != OP_NF4_K || p.seg[0].A.kind != OP_BF16_K) return false;
  if (p.accumulate || p.out_f32 || p.out_trans) return false;
  if (p.residual && (p.ldr % 8 != 0 || !aligned16(p.residual))) return false;
  if (p.seg[0].K % 1024 != 0 || p.seg[0].B.row_lo > 0 || p.seg[0].B.row_hi < p.N) return false;
  if (p.rope_cols > 0 && (p.residual || p.rope_d != 128 || p.rope_rl != 0 || p.rope_S % TsCfg::BT != 0 ||
                         p.M % TsCfg::BT != 0 || p.rope_cols % TsCfg::BW != 0))
    return false;
  for (int s = 0; s < p.nseg; ++s) {
    const GemmSeg& sg = p.seg[s];
    if (sg.A.scale != 1.f || sg.B.scale != 1.f) return false;
    if (s == 0) continue;
    if (sg.K <= 0 || sg.K % 8 != 0 || sg.A.kind != OP_BF16_K || sg.B.kind != OP_BF16_K) return false;
    if (sg.B.ld % 8 != 0 || !aligned16(sg.B.ptr)) return false;
  }
  const long long tiles = static_cast<long long>((p.N + TsCfg::BW - 1) / TsCfg::BW) * ((p.M + TsCfg::BT - 1) / TsCfg::BT);
  return tiles >= TS_MIN_TILES;
}
// Sets up the descriptors and launches gemm_ts_kernel; false (nothing launched) when a
// descriptor cannot be encoded, so the caller takes the shared-memory kernel.
bool launch_ts(GemmParams& p, cudaStream_t st, cudaError_t* err) {
  if (!setup_raw_tma(p, TsCfg::BW)) return false;
  for (int s = 0; s < p.nseg; ++s) {
    const GemmSeg& sg = p.seg[s];
    if (sg.K > 0 && !encode_kmajor_bf16(&p.tmapA[s], sg.A.ptr, sg.K, p.M, sg.A.ld, TsCfg::BT)) return false;
  }
  if (p.residual && !encode_cached(&p.tmapB[0], p.residual, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                                   static_cast<unsigned long long>(p.N), static_cast<unsigned long long>(p.M),
                                   static_cast<unsigned long long>(p.ldr) * 2, TsCfg::BW, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
    return false;
  if (p.rope_cols > 0) {
    for (int t = 0; t < 2; ++t)
      if (!encode_cached(&p.tmapB[1 + t], t ? p.rope_sin : p.rope_cos, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 64,
                         static_cast<unsigned long long>(p.rope_S), 64 * 4, 64, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
        return false;
  }
  p.raw_tma = 1;
  p.bn = TsCfg::BW;
  p.splits = 1;
  p.sk_ctas = 0;
  static std::atomic<int> attr_done{0};
  if (!attr_done.load()) {
    const cudaError_t e = cudaFuncSetAttribute(gemm_ts_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               TsCfg::SMEM_BYTES);
    if (e != cudaSuccess) {
      *err = e;
      return true;
    }
    attr_done.store(1);
  }
  const dim3 grid((p.N + TsCfg::BW - 1) / TsCfg::BW, (p.M + TsCfg::BT - 1) / TsCfg::BT, 1);
  gemm_ts_kernel<<<grid, GEMM_THREADS, TsCfg::SMEM_BYTES, st>>>(p);
  *err = cudaGetLastError();
  return true;
}

// SMs of the current device (stream-K spreads a GEMM over one CTA per SM)
int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int n = cached[dev].load();
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev].store(n);
  }
  return n;
}
// SOUP_GEMM_STREAMK=0 keeps every GEMM on whole tiles (for comparisons)
bool sk_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("SOUP_GEMM_STREAMK");
    return !(e && e[0] == '0');
  }();
  return on;
}

bool operand_ok(const Operand& op, int K) {
  switch (op.kind) {
    case OP_BF16_K:
      return aligned16(op.ptr) && op.ld % 8 == 0 && K % 8 == 0;
    case OP_F32_K:
      return aligned16(op.ptr) && op.ld % 4 == 0 && K % 8 == 0;
    case OP_BF16_MN:
      return aligned16(op.ptr) && op.ld % 8 == 0;
    case OP_F32_MN:
      return aligned16(op.ptr) && op.ld % 4 == 0;
    case OP_NF4_K:
      return K % 8 == 0;
    case OP_NF4_MN:
      return true;
    default:
      return false;
  }
}

bool is_mn(int kind) { return kind == OP_BF16_MN || kind == OP_F32_MN || kind == OP_NF4_MN; }

}  // namespace

bool tma_encode_bf16_sw128_planes(CUtensorMap* map, const void* ptr, unsigned long long rows, unsigned long long planes,
                                  unsigned long long row_bytes, unsigned box_rows, unsigned box_planes) {
  if (rows == 0 || planes == 0 || (reinterpret_cast<uintptr_t>(ptr) & 15u) || (row_bytes & 15u)) return false;
  return encode_cached(map, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, rows, row_bytes, 64, box_rows,
                       CU_TENSOR_MAP_SWIZZLE_128B, planes, 128, box_planes);
}

bool tma_encode_bf16_sw128(CUtensorMap* map, const void* ptr, unsigned long long inner, unsigned long long outer,
                           unsigned long long row_bytes, unsigned box_inner, unsigned box_outer) {
  if (inner == 0 || outer == 0 || (reinterpret_cast<uintptr_t>(ptr) & 15u) || (row_bytes & 15u)) return false;
  return encode_cached(map, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, inner, outer, row_bytes, box_inner, box_outer,
                       CU_TENSOR_MAP_SWIZZLE_128B);
}

GemmPlan gemm_plan(const GemmParams& p, int sms, bool stream_k_allowed) {
  GemmPlan pl{};
  if (sms < 1) sms = 148;
  long long nkb = 0;
  for (int s = 0; s < p.nseg; ++s)
    if (p.seg[s].K > 0) nkb += (p.seg[s].K + BK - 1) / BK;
  // Tile choice: MT 128-row halves x BN columns.  Time ~ waves x per-tile time, with the per-tile
  // time proportional to the k-blocks and a per-k-block cost measured on B200 for each tile
  // shape (NF4 GEMMs at M = 512 and 2048): 2x128 50, 1x256 60, 1x128 38, 2x64 47, 1x64 36.
  // GEMMs without an NF4 operand have no decode: a k-block costs about the issuing thread's
  // MT x 4 tcgen05.mma instructions (~100 cycles each for N <= 128), so the skinny LoRA GEMMs
  // (N <= 192) prefer one 128-row tile; the 1x256 tile (N = 256 instructions, 3 stages) ran
  // the lm_head GEMMs 25 % slower than 2x128, hence its cost.
  bool has_nf4 = false;
  for (int s = 0; s < p.nseg; ++s)
    if (p.seg[s].K > 0 && (p.seg[s].B.kind == OP_NF4_K || p.seg[s].B.kind == OP_NF4_MN)) has_nf4 = true;
  // a RoPE epilogue needs whole tiles that hold whole heads and never straddle the RoPE range
  const bool rope = p.rope_cols > 0;
  const int cand[5][2] = {{2, 128}, {1, 256}, {1, 128}, {2, 64}, {1, 64}};
  const double unit_nf4[5] = {50.0, 60.0, 38.0, 47.0, 36.0};
  const double unit_bf16[5] = {50.0, 60.0, 36.0, 64.0, 36.0};
  const double* unit = has_nf4 ? unit_nf4 : unit_bf16;
  // split-K for grids that leave SMs idle (the skinny LoRA GEMMs; never NF4): up to two waves
  // of CTAs, at least 4 k-blocks per split (a CTA of these runs at the issuing thread's rate,
  // so spreading K shortens the GEMM).  The cost below includes the split and the sum of the
  // partials (the tile's last CTA for up to 4, else the wide reduction kernel).
  auto split_cost = [&](long long tiles, long long sp, double u) {
    const long long waves = (tiles * sp + sms - 1) / sms;
    return static_cast<double>(waves) * (static_cast<double>((nkb + sp - 1) / sp) + 2.0) * u +
           (sp > 4 ? 360.0 : (sp > 1 ? 130.0 : 0.0));
  };
  // the split count: the cheapest of 1..4 (summed by the tile's last CTA) and the widest
  // allowed (summed by the reduction kernel).  The sums' costs are fitted to the LoRA shapes
  // timed on B200 (k-block ~1 us at these tiles): the reduction kernel ~10 us, the last CTA's
  // sum of up to 4 partials ~4 us; u of q|k|v (N 192, K 4096) at 512 rows ran 17.5 us with 16
  // splits and 23.5 with 4, at 2048 rows 35.5 with 10 and 23.6 with 4
  auto split_for = [&](long long tiles, double u) -> long long {
    if (!p.workspace || !p.tile_counters || has_nf4 || tiles >= 100 || nkb < 16 || tiles > p.n_counters) return 1;
    long long mx = (2 * sms + tiles - 1) / tiles;
    mx = std::min<long long>(mx, nkb / 4);
    mx = std::min<long long>(mx, 32);
    while (mx > 1 && static_cast<unsigned long long>(mx) * p.M * p.N * 4ull > p.ws_bytes) --mx;
    if (mx < 1) mx = 1;
    long long best_sp = 1;
    double best_c = split_cost(tiles, 1, u);
    const long long cands[5] = {2, 3, 4, mx, 0};
    for (int i = 0; cands[i] > 0; ++i) {
      const long long sp = cands[i];
      if (sp > mx) continue;
      const double c = split_cost(tiles, sp, u);
      if (c < best_c * 0.999) {
        best_c = c;
        best_sp = sp;
      }
    }
    return best_sp;
  };
  int MT = 1, BN = 128;
  double best = 1e300;
  for (int ci = 0; ci < 5; ++ci) {
    const int mt = cand[ci][0], bn = cand[ci][1];
    if (mt == 2 && p.M <= UM) continue;
    if (bn > 64 && p.N <= 64) continue;
    if (bn > 128 && p.N <= 128) continue;
    if (rope && (bn % p.rope_d != 0 || p.rope_cols % bn != 0)) continue;
    const long long tl = static_cast<long long>((p.N + bn - 1) / bn) * ((p.M + UM * mt - 1) / (UM * mt));
    const long long sp = split_for(tl, unit[ci]);
    const double cost = split_cost(tl, sp, unit[ci]);
    if (cost < best * 0.999) {
      best = cost;
      MT = mt;
      BN = bn;
    }
  }
  // Stream-K for NF4 GEMMs whose whole-tile grid leaves SMs idle (gate|up forward at 512
  // rows: 448 CTAs = 3.03 waves; its dX: 128 CTAs of 450 k-blocks on 148 SMs): the 256x128
  // tile (the cheapest per output), every k-block of every tile spread evenly over one CTA per
  // SM.  Its cost adds ~4 k-blocks per piece (the epilogue between pieces, the pipeline
  // refill) and ~24 for the partial tiles' shares (stored, then summed by all threads at the
  // end).  Measured on the 8B projections at 512 rows: gate|up dX 200 -> 155 us, forward
  // 176 -> 164, down forward 106 -> 97; the short q|k|v and o GEMMs (28-42 k-blocks per CTA)
  // ran 20-40 % slower, as did every GEMM at 2048 rows, where whole tiles already fill 86-93 %
  // of the SMs and ran faster per k-block: so at most two 256-row M-tiles.  Only when every
  // N-tile has the same active segments (the flattened k-block count is then tiles x k-blocks
  // per tile) and a tile is cut into at most 4 shares.
  if (has_nf4 && !rope && p.workspace && p.tile_counters && stream_k_allowed && p.M <= 2 * UM * 2) {
    const int mt = p.M > UM ? 2 : 1, bn = 128, bm = UM * mt;
    const int tiles_n = (p.N + bn - 1) / bn, tiles_m = (p.M + bm - 1) / bm;
    int nkt = -1;
    bool uniform = true;
    for (int tn = 0; tn < tiles_n && uniform; ++tn) {
      int nk = 0;
      for (int s = 0; s < p.nseg; ++s) {
        const GemmSeg& sg = p.seg[s];
        if (sg.K > 0 && sg.B.row_lo < tn * bn + bn && sg.B.row_hi > tn * bn) nk += (sg.K + BK - 1) / BK;
      }
      if (nkt < 0) nkt = nk;
      uniform = nk == nkt;
    }
    const int G = sms;
    const long long T = static_cast<long long>(tiles_n) * tiles_m;
    const long long W = T * (nkt > 0 ? nkt : 0);
    const long long per = G > 0 ? W / G : 0;
    const size_t ws_need = static_cast<size_t>(2) * G * bm * bn * sizeof(float);
    if (uniform && nkt > 0 && per >= 8 && T <= p.n_counters && ws_need <= p.ws_bytes &&
        nkt <= 3 * per + 1) {  // at most 4 shares per tile
      const int ci = mt == 2 ? 0 : 2;  // 2x128 or 1x128 in the cost table
      const long long pieces = (per + nkt - 1) / nkt + 1;
      const double cost_sk = (static_cast<double>(per) + 2.0 + 4.0 * pieces + 24.0) * unit[ci];
      if (cost_sk < 0.95 * best) {
        MT = mt;
        BN = bn;
        pl.sk_ctas = G;
        pl.sk_tiles = static_cast<int>(T);
        pl.sk_tiles_m = tiles_m;
        pl.sk_nkt = nkt;
      }
    }
  }
  pl.mt = MT;
  pl.bn = BN;
  // NF4 GEMMs keep whole K (the 96-tile q|k|v GEMM ran 105 us split four ways, 65 us whole)
  const int BM = UM * MT;
  const long long tiles = static_cast<long long>((p.N + BN - 1) / BN) * ((p.M + BM - 1) / BM);
  int ci_chosen = 0;
  for (int ci = 0; ci < 5; ++ci)
    if (cand[ci][0] == MT && cand[ci][1] == BN) ci_chosen = ci;
  pl.splits = (has_nf4 || rope || pl.sk_ctas > 0) ? 1 : static_cast<int>(split_for(tiles, unit[ci_chosen]));
  // up to 4 partials the tile's last CTA sums them; more run through the wide reduction
  // kernel (measured: 16-32 partials summed by one CTA per tile cost more than the launch)
  pl.fused_reduce = pl.splits <= 4 ? 1 : 0;
  return pl;
}

cudaError_t gemm_launch(const GemmParams& p_in, cudaStream_t st) {
  if (p_in.M <= 0 || p_in.N <= 0) return cudaSuccess;
  GemmParams p = p_in;
  if (p.N % 8 != 0 || p.nseg < 1 || p.nseg > GEMM_MAX_SEG) return cudaErrorInvalidValue;
  if (!aligned16(p.out)) return cudaErrorInvalidValue;
  if (p.rope_cols > 0 &&
      (p.out_f32 || p.out_trans || p.residual || p.accumulate || !p.rope_cos || !p.rope_sin || p.rope_S <= 0 ||
       (p.rope_d != 64 && p.rope_d != 128) || p.rope_cols % p.rope_d != 0 || p.rope_cols > p.N))
    return cudaErrorInvalidValue;
  if (p.out_trans) {
    if (p.residual) return cudaErrorInvalidValue;
  } else {
    if (p.ldo % 8 != 0) return cudaErrorInvalidValue;
    if (p.residual && (!aligned16(p.residual) || p.ldr % 8 != 0)) return cudaErrorInvalidValue;
  }
  for (int s = 0; s < p.nseg; ++s) {
    GemmSeg& sg = p.seg[s];
    p.a_mode[s] = 0;
    p.b_mode[s] = 0;
    p.b_row0[s] = 0;
    if (sg.K < 0) return cudaErrorInvalidValue;
    if (sg.K == 0) continue;
    if (!operand_ok(sg.A, sg.K) || !operand_ok(sg.B, sg.K)) return cudaErrorInvalidValue;
    if (is_mn(sg.A.kind) && p.M % 8 != 0) return cudaErrorInvalidValue;
    if (sg.A.kind == OP_NF4_K || sg.A.kind == OP_NF4_MN) return cudaErrorInvalidValue;  // NF4 only as B
    if (sg.B.kind == OP_NF4_K && (p.nf4.cols % 8 != 0 || sg.K > p.nf4.cols)) return cudaErrorInvalidValue;
    if (sg.B.kind == OP_NF4_MN && (p.nf4.cols % 8 != 0 || p.N > p.nf4.cols)) return cudaErrorInvalidValue;
  }
  if (ts_applicable(p)) {
    cudaError_t e = cudaSuccess;
    if (launch_ts(p, st, &e)) {
      ++g_kernel_launches;
      return e;
    }
  }
  const GemmPlan pl = gemm_plan(p, sm_count(), sk_enabled());
  const int MT = pl.mt, BN = pl.bn;
  p.sk_ctas = pl.sk_ctas;
  p.sk_tiles = pl.sk_tiles;
  p.sk_tiles_m = pl.sk_tiles_m;
  p.sk_nkt = pl.sk_nkt;
  const int BM = UM * MT;  // A rows per CTA
  const int BNB = BN;      // B rows per CTA
  p.bn = BNB;
  p.raw_tma = setup_raw_tma(p, BNB) ? 1 : 0;
  if (tma_operands_allowed()) {
    for (int s = 0; s < p.nseg; ++s) {
      GemmSeg& sg = p.seg[s];
      if (sg.K <= 0) continue;
      if (sg.A.kind == OP_BF16_K)
        p.a_mode[s] = encode_kmajor_bf16(&p.tmapA[s], sg.A.ptr, sg.K, p.M, sg.A.ld, BM) ? 1 : 0;
      else if (sg.A.kind == OP_BF16_MN)
        p.a_mode[s] = encode_mnmajor_bf16(&p.tmapA[s], sg.A.ptr, p.M, sg.K, sg.A.ld) ? 2 : 0;
      if (sg.B.kind == OP_BF16_K) {
        // a block-diagonal window [row_lo, row_hi) becomes the descriptor's whole extent, so
        // rows outside it read as zero through the TMA's out-of-bounds fill
        const int lo = std::max(0, sg.B.row_lo), hi = std::min(p.N, sg.B.row_hi);
        if (hi > lo) {
          const void* base = static_cast<const uint16_t*>(sg.B.ptr) + static_cast<long long>(lo) * sg.B.ld;
          if (encode_kmajor_bf16(&p.tmapB[s], base, sg.K, hi - lo, sg.B.ld, BNB)) {
            p.b_mode[s] = 1;
            p.b_row0[s] = lo;
          }
        }
      } else if (sg.B.kind == OP_BF16_MN && sg.B.row_lo <= 0 && sg.B.row_hi >= p.N) {
        p.b_mode[s] = encode_mnmajor_bf16(&p.tmapB[s], sg.B.ptr, p.N, sg.K, sg.B.ld) ? 2 : 0;
      }
    }
  } else {
    for (int s = 0; s < p.nseg; ++s)
      if (p.seg[s].K > 0 && p.seg[s].A.kind == OP_BF16_K)
        p.a_mode[s] = encode_kmajor_bf16(&p.tmapA[s], p.seg[s].A.ptr, p.seg[s].K, p.M, p.seg[s].A.ld, BM) ? 1 : 0;
  }
  p.splits = pl.splits;
  p.fused_reduce = pl.fused_reduce;
  cudaError_t e;
  if (p.sk_ctas > 0)
    e = (MT == 2) ? launch_tile<2, 128, true>(p, st) : launch_tile<1, 128, true>(p, st);
  else if (MT == 2)
    e = (BN == 64) ? launch_tile<2, 64>(p, st) : launch_tile<2, 128>(p, st);
  else
    e = (BN == 64) ? launch_tile<1, 64>(p, st) : (BN == 128 ? launch_tile<1, 128>(p, st) : launch_tile<1, 256>(p, st));
  ++g_kernel_launches;
  return e;
}

}  // namespace soup
