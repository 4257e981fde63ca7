// Tensor-core GEMM for sm_100a: C[M,N] = sum over segments of A_s[M,K_s] . B_s[N,K_s]^T.
//
// This single kernel carries every contraction of the decoder layer:
//   * forward  y = x W^T + s (x A^T) B^T : segment 0 streams the NF4 weight (dequantised by the
//     producer warps), later segments are the LoRA branch appended as extra K-blocks;
//   * backward dx = dy W + s (dy B) A     : the same NF4 weight read transposed;
//   * LoRA grads, lm_head forward/backward: plain bf16 / fp32 operands.
//
// Roles (384 threads, one CTA per 128 x BN output tile):
//   warps 0-7  producers: global -> registers -> (NF4 LUT dequant | fp32->bf16 | copy) ->
//              shared memory in the 128-byte-swizzled K-major layout the tensor core reads;
//   warp 8     allocates the TMEM accumulator; lane 0 issues tcgen05.mma (M=128, N=BN, K=16)
//              and tcgen05.commit to release stages;
//   warps 8-11 epilogue: tcgen05.ld rows out of TMEM, scale, add residual / old value, store.
// A STAGES-deep ring of (A,B) tiles with full/empty mbarriers overlaps loads with MMAs.
//
// NF4 decode follows the double-quantised format: mhat = fp32(fp32(q8 * s2) + mean),
// w = bf16_rn(fp32(code_value * mhat)), one float32 multiply per element, codebook read from
// a 16-entry shared-memory table.
#include "common.cuh"
#include "internal.h"

#include <atomic>

namespace soup {

namespace {

constexpr int GEMM_THREADS = 384;
constexpr int PRODUCER_THREADS = 256;
constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = 128 bytes = one swizzle row

template <int BN>
struct GemmCfg {
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (BN >= 256) ? 4 : (BN >= 128 ? 5 : 6);
  static constexpr int CTRL_BYTES = 512;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + CTRL_BYTES;
};

// ---------------------------------------------------------------- tcgen05 wrappers
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row core groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(1) << 16;                  // leading byte offset (unused with this swizzle)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;          // stride byte offset: next 8-row group
  d |= static_cast<uint64_t>(1) << 46;                  // descriptor version for sm_100
  d |= static_cast<uint64_t>(2) << 61;                  // swizzle mode: 128 B
  return d;
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> f32, both operands K-major, M = 128.
template <int BN>
__device__ __forceinline__ uint32_t idesc_bf16_f32() {
  return (1u << 4)                                 // D format f32
         | (1u << 7)                               // A format bf16
         | (1u << 10)                              // B format bf16
         | (static_cast<uint32_t>(BN >> 3) << 17)  // N / 8
         | (static_cast<uint32_t>(BM >> 4) << 24); // M / 16
}

// ---------------------------------------------------------------- operand fetch
__device__ __forceinline__ float nf4_mhat(const NF4Seg& sg, long long blk) {
  const float s2 = __ldg(sg.scales + (blk >> 8));
  const float q = static_cast<float>(__ldg(sg.q8 + blk));
  return __fadd_rn(__fmul_rn(q, s2), __ldg(sg.mean));
}

// 8 consecutive columns [wc, wc+8) of NF4 row wr as 8 bf16 (wc multiple of 8, in range).
__device__ __forceinline__ uint4 nf4_chunk8(const NF4Group& g, const float* lut, int wr, int wc) {
  int s = 0;
  if (g.nseg > 1 && wr >= g.seg[1].row_begin) s = 1;
  if (g.nseg > 2 && wr >= g.seg[2].row_begin) s = 2;
  const NF4Seg& sg = g.seg[s];
  const long long flat = static_cast<long long>(wr - sg.row_begin) * g.cols + wc;
  const float mh = nf4_mhat(sg, flat >> 6);
  const uint32_t c = __ldg(reinterpret_cast<const uint32_t*>(sg.codes + (flat >> 1)));
  uint4 o;
  o.x = pack_bf16x2(__fmul_rn(lut[c & 15u], mh), __fmul_rn(lut[(c >> 4) & 15u], mh));
  o.y = pack_bf16x2(__fmul_rn(lut[(c >> 8) & 15u], mh), __fmul_rn(lut[(c >> 12) & 15u], mh));
  o.z = pack_bf16x2(__fmul_rn(lut[(c >> 16) & 15u], mh), __fmul_rn(lut[(c >> 20) & 15u], mh));
  o.w = pack_bf16x2(__fmul_rn(lut[(c >> 24) & 15u], mh), __fmul_rn(lut[c >> 28], mh));
  return o;
}

__device__ __forceinline__ uint4 fetch_kmajor(const Operand& op, const NF4Group& g, const float* lut, int r, int k) {
  switch (op.kind) {
    case OP_BF16_K:
      return __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(op.ptr) + r * op.ld + k));
    case OP_F32_K: {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(op.ptr) + r * op.ld + k);
      const float4 a = __ldg(src), b = __ldg(src + 1);
      const float s = op.scale;
      uint4 o;
      o.x = pack_bf16x2(a.x * s, a.y * s);
      o.y = pack_bf16x2(a.z * s, a.w * s);
      o.z = pack_bf16x2(b.x * s, b.y * s);
      o.w = pack_bf16x2(b.z * s, b.w * s);
      return o;
    }
    default:  // OP_NF4_K
      return nf4_chunk8(g, lut, r, k);
  }
}

// 8 consecutive rows [r, r+8) at reduction index k, as 8 bf16 (zero when k >= K).
__device__ __forceinline__ uint4 fetch_mn8(const Operand& op, const NF4Group& g, const float* lut, int r, int k,
                                           int K) {
  if (k >= K) return make_uint4(0, 0, 0, 0);
  switch (op.kind) {
    case OP_BF16_MN:
      return __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(op.ptr) + k * op.ld + r));
    case OP_F32_MN: {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(op.ptr) + k * op.ld + r);
      const float4 a = __ldg(src), b = __ldg(src + 1);
      const float s = op.scale;
      uint4 o;
      o.x = pack_bf16x2(a.x * s, a.y * s);
      o.y = pack_bf16x2(a.z * s, a.w * s);
      o.z = pack_bf16x2(b.x * s, b.y * s);
      o.w = pack_bf16x2(b.z * s, b.w * s);
      return o;
    }
    default:  // OP_NF4_MN: W[k, r..r+7]
      return nf4_chunk8(g, lut, k, r);
  }
}

__device__ __forceinline__ uint32_t swz_off(int r, int chunk) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((chunk ^ (r & 7)) << 4));
}

// Fill one ROWS x 64 tile of an operand into swizzled shared memory.
template <int ROWS>
__device__ __forceinline__ void load_tile(const Operand& op, const NF4Group& g, const float* lut, int K, int row0,
                                          int nrows, int k0, uint8_t* tile, int ptid) {
  const bool kmajor = (op.kind == OP_BF16_K || op.kind == OP_F32_K || op.kind == OP_NF4_K);
  if (kmajor) {
#pragma unroll 2
    for (int c = ptid; c < ROWS * 8; c += PRODUCER_THREADS) {
      const int rr = c >> 3, kc = c & 7;
      const int row = row0 + rr, k = k0 + kc * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (row < nrows && row >= op.row_lo && row < op.row_hi && k < K) v = fetch_kmajor(op, g, lut, row, k);
      *reinterpret_cast<uint4*>(tile + swz_off(rr, kc)) = v;
    }
  } else {
    // units of 8 rows x 2 consecutive k; 32 k-pairs per warp pass keep the 4-byte stores conflict-free
    for (int u = ptid; u < (ROWS / 8) * 32; u += PRODUCER_THREADS) {
      const int kp = u & 31, grp = u >> 5;
      const int rr0 = grp * 8, row = row0 + rr0, k = k0 + kp * 2;
      uint4 x0 = make_uint4(0, 0, 0, 0), x1 = make_uint4(0, 0, 0, 0);
      if (row < nrows && row >= op.row_lo && row < op.row_hi) {
        x0 = fetch_mn8(op, g, lut, row, k, K);
        x1 = fetch_mn8(op, g, lut, row, k + 1, K);
      }
      const uint32_t a[4] = {x0.x, x0.y, x0.z, x0.w};
      const uint32_t b[4] = {x1.x, x1.y, x1.z, x1.w};
      const uint32_t inchunk = (kp & 3) * 4;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t lo = __byte_perm(a[j], b[j], 0x5410);  // (row 2j: k, k+1)
        const uint32_t hi = __byte_perm(a[j], b[j], 0x7632);  // (row 2j+1: k, k+1)
        *reinterpret_cast<uint32_t*>(tile + swz_off(rr0 + 2 * j, kp >> 2) + inchunk) = lo;
        *reinterpret_cast<uint32_t*>(tile + swz_off(rr0 + 2 * j + 1, kp >> 2) + inchunk) = hi;
      }
    }
  }
}

__device__ __forceinline__ bool seg_active(const GemmSeg& s, int n0, int bn) {
  if (s.K <= 0) return false;
  return s.B.row_lo < n0 + bn && s.B.row_hi > n0;
}

// ---------------------------------------------------------------- the kernel
template <int BN>
__global__ void __launch_bounds__(GEMM_THREADS, 1) gemm_tc_kernel(const __grid_constant__ GemmParams p) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* ctrl = base + C::STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + C::STAGES;
  uint64_t* done = empty + C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* lut = reinterpret_cast<float*>(ctrl + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], PRODUCER_THREADS / 32);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (threadIdx.x < 16) lut[threadIdx.x] = p.lut[threadIdx.x];
  if (warp == 8) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 8) {
    // ------------------------------------------------ producers
    const int ptid = threadIdx.x;
    int kb = 0;
    for (int s = 0; s < p.nseg; ++s) {
      const GemmSeg& sg = p.seg[s];
      if (!seg_active(sg, n0, BN)) continue;
      const int nk = (sg.K + BK - 1) / BK;
      for (int kk = 0; kk < nk; ++kk, ++kb) {
        const int st = kb % C::STAGES;
        const uint32_t ph = static_cast<uint32_t>(kb / C::STAGES) & 1u;
        mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, p.err);
        uint8_t* As = base + st * C::STAGE_BYTES;
        uint8_t* Bs = As + C::A_BYTES;
        load_tile<BM>(sg.A, p.nf4, lut, sg.K, m0, p.M, kk * BK, As, ptid);
        load_tile<BN>(sg.B, p.nf4, lut, sg.K, n0, p.N, kk * BK, Bs, ptid);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[st]);
      }
    }
  } else {
    if (warp == 8 && lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16_f32<BN>();
      int kb = 0;
      for (int s = 0; s < p.nseg; ++s) {
        const GemmSeg& sg = p.seg[s];
        if (!seg_active(sg, n0, BN)) continue;
        const int nk = (sg.K + BK - 1) / BK;
        for (int kk = 0; kk < nk; ++kk, ++kb) {
          const int st = kb % C::STAGES;
          const uint32_t ph = static_cast<uint32_t>(kb / C::STAGES) & 1u;
          mbar_wait_bounded(&full[st], ph, abort_flag, p.err);
          tc_fence_after();
          const uint32_t a_addr = smem_u32(base + st * C::STAGE_BYTES);
          const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
          for (int j = 0; j < BK / 16; ++j) {
            tc_mma_f16(tmem, sw128_kmajor_desc(a_addr + j * 32), sw128_kmajor_desc(b_addr + j * 32), idesc,
                       (kb > 0 || j > 0) ? 1u : 0u);
          }
          tc_commit(&empty[st]);
        }
      }
      tc_commit(done);
    }
    __syncwarp();
    // ------------------------------------------------ epilogue (warps 8..11 = TMEM lane quarters 0..3)
    const int q = warp - 8;
    mbar_wait_bounded(done, 0u, abort_flag, p.err);
    tc_fence_after();
    bool any_k = false;
    for (int s = 0; s < p.nseg; ++s) any_k |= seg_active(p.seg[s], n0, BN);
    const int row = m0 + q * 32 + lane;
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(cc), r);
      tmem_ld_wait();
      if (row >= p.M) continue;
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8) {
        const int col = n0 + cc + g8 * 8;
        if (col >= p.N) break;
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = any_k ? p.alpha * __uint_as_float(r[g8 * 8 + j]) : 0.f;
        if (!p.out_trans) {
          if (p.residual) {
            const uint4 rv =
                *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.residual) + row * p.ldr + col);
            const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 f = unpack_bf16x2(rw[j]);
              v[2 * j] += f.x;
              v[2 * j + 1] += f.y;
            }
          }
          if (p.out_f32) {
            float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * p.ldo + col);
            if (p.accumulate) {
              const float4 a = o[0], b = o[1];
              v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
              v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
            }
            o[0] = make_float4(v[0], v[1], v[2], v[3]);
            o[1] = make_float4(v[4], v[5], v[6], v[7]);
          } else {
            uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * p.ldo + col);
            if (p.accumulate) {
              const uint4 a = *o;
              const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float2 f = unpack_bf16x2(aw[j]);
                v[2 * j] += f.x;
                v[2 * j + 1] += f.y;
              }
            }
            *o = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                            pack_bf16x2(v[6], v[7]));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const long long idx = static_cast<long long>(col + j) * p.ldo + row;
            if (p.out_f32) {
              float* o = static_cast<float*>(p.out) + idx;
              *o = p.accumulate ? (*o + v[j]) : v[j];
            } else {
              uint16_t* o = static_cast<uint16_t*>(p.out) + idx;
              float w = v[j];
              if (p.accumulate) w += bf16_to_f32(*o);
              const __nv_bfloat16 b = __float2bfloat16_rn(w);
              *o = *reinterpret_cast<const uint16_t*>(&b);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

template <int BN>
cudaError_t launch_bn(const GemmParams& p, cudaStream_t st) {
  using C = GemmCfg<BN>;
  static std::atomic<int> attr_done{0};
  if (!attr_done.load()) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done.store(1);
  }
  dim3 grid((p.N + BN - 1) / BN, (p.M + BM - 1) / BM);
  gemm_tc_kernel<BN><<<grid, GEMM_THREADS, C::SMEM_BYTES, st>>>(p);
  return cudaGetLastError();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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

cudaError_t gemm_launch(const GemmParams& p, cudaStream_t st) {
  if (p.M <= 0 || p.N <= 0) return cudaSuccess;
  if (p.N % 8 != 0 || p.nseg < 1 || p.nseg > GEMM_MAX_SEG) return cudaErrorInvalidValue;
  if (!aligned16(p.out)) return cudaErrorInvalidValue;
  if (p.out_trans) {
    if (p.residual) return cudaErrorInvalidValue;
  } else {
    if (p.ldo % 8 != 0) return cudaErrorInvalidValue;
    if (p.residual && (!aligned16(p.residual) || p.ldr % 8 != 0)) return cudaErrorInvalidValue;
  }
  for (int s = 0; s < p.nseg; ++s) {
    const GemmSeg& sg = p.seg[s];
    if (sg.K < 0) return cudaErrorInvalidValue;
    if (sg.K == 0) continue;
    if (!operand_ok(sg.A, sg.K) || !operand_ok(sg.B, sg.K)) return cudaErrorInvalidValue;
    if (is_mn(sg.A.kind) && p.M % 8 != 0) return cudaErrorInvalidValue;
    if ((sg.A.kind == OP_NF4_K || sg.A.kind == OP_NF4_MN)) return cudaErrorInvalidValue;  // NF4 only as B
    if (sg.B.kind == OP_NF4_K && (p.nf4.cols % 8 != 0 || sg.K > p.nf4.cols)) return cudaErrorInvalidValue;
    if (sg.B.kind == OP_NF4_MN && (p.nf4.cols % 8 != 0 || p.N > p.nf4.cols)) return cudaErrorInvalidValue;
  }
  cudaError_t e;
  if (p.N <= 64)
    e = launch_bn<64>(p, st);
  else if (p.N <= 128 || static_cast<long long>((p.N + 255) / 256) * ((p.M + 127) / 128) < 148)
    e = launch_bn<128>(p, st);
  else
    e = launch_bn<256>(p, st);
  ++g_kernel_launches;
  return e;
}

}  // namespace soup
