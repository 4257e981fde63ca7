// NF4 quantiser (create-time, untimed) and standalone NF4 -> bf16 dequantiser.
//
// Format (one tensor, row-major flattened, n elements):
//   blocks of 64 consecutive elements: absmax m = max |w|; code = argmin_j |w/m - c_j| taken in
//   float64 with the lowest index on ties (m = 0 gives the code of 0.0); element 2i in the low
//   nibble of byte i, a trailing odd element leaves the high nibble 0;
//   absmax double quantisation: mean = float32(sequential float64 sum of m / nb); per group of
//   256 blocks s2 = float32(max |m - mean| / 127) (1 if that is 0), q8 = clamp(rint((m - mean)/s2))
//   in float64; the dequantiser reconstructs mhat = fp32(fp32(q8*s2) + mean) and
//   w = bf16_rn(fp32(c_q * mhat)).
// The integer decisions (codes, q8) are taken in float64 on exact inputs, so they are
// reproducible bit for bit by any implementation of the same definition.
#include "../../include/soup.h"
#include "common.cuh"
#include "internal.h"

#include <mutex>

namespace soup {

namespace {

// One warp per 64-element block: lane l owns elements 2l and 2l+1.
__global__ void nf4_block_codes_kernel(const float* __restrict__ w, long long n, long long nb, uint8_t* __restrict__ codes,
                                       float* __restrict__ absmax, const LUT16 lut) {
  const long long blk = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (blk >= nb) return;
  const long long e0 = blk * 64 + 2 * lane;
  const float w0 = (e0 < n) ? w[e0] : 0.f;
  const float w1 = (e0 + 1 < n) ? w[e0 + 1] : 0.f;
  float m = fmaxf(fabsf(w0), fabsf(w1));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) absmax[blk] = m;
  int q[2] = {7, 7};
  if (m > 0.f) {
    const double md = static_cast<double>(m);
    const float wv[2] = {w0, w1};
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const double r = static_cast<double>(wv[t]) / md;
      int best = 0;
      double bd = fabs(r - static_cast<double>(lut.v[0]));
#pragma unroll
      for (int j = 1; j < 16; ++j) {
        const double dd = fabs(r - static_cast<double>(lut.v[j]));
        if (dd < bd) {
          bd = dd;
          best = j;
        }
      }
      q[t] = best;
    }
  } else {
    // code of 0.0 (index 7 in the ascending NF4 codebook)
    int z = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (lut.v[j] == 0.f) z = j;
    q[0] = q[1] = z;
  }
  if (e0 < n) {
    const int hi = (e0 + 1 < n) ? q[1] : 0;
    codes[e0 >> 1] = static_cast<uint8_t>(q[0] | (hi << 4));
  }
}

// Sequential float64 sum of the absmax (the format's definition of the mean).  One block:
// tiles are staged through shared memory, thread 0 adds them in index order.
__global__ void nf4_mean_kernel(const float* __restrict__ absmax, long long nb, float* __restrict__ mean) {
  __shared__ float tile[1024];
  double acc = 0.0;
  for (long long base = 0; base < nb; base += 1024) {
    const long long i = base + threadIdx.x;
    tile[threadIdx.x] = (i < nb) ? absmax[i] : 0.f;
    __syncthreads();
    if (threadIdx.x == 0) {
      const int cnt = static_cast<int>((nb - base) < 1024 ? (nb - base) : 1024);
      for (int j = 0; j < cnt; ++j) acc += static_cast<double>(tile[j]);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) *mean = static_cast<float>(acc / static_cast<double>(nb));
}

// One warp per group of 256 blocks: lane l owns blocks 8l..8l+7 of the group.
__global__ void nf4_dq_kernel(const float* __restrict__ absmax, long long nb, const float* __restrict__ mean,
                              int8_t* __restrict__ q8, float* __restrict__ scales) {
  const long long grp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long ng = (nb + 255) / 256;
  if (grp >= ng) return;
  const double mu = static_cast<double>(*mean);
  double d[8];
  double amax = 0.0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const long long b = grp * 256 + lane * 8 + j;
    d[j] = (b < nb) ? static_cast<double>(absmax[b]) - mu : 0.0;
    if (b < nb) amax = fmax(amax, fabs(d[j]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s2 = (amax > 0.0) ? static_cast<float>(amax / 127.0) : 1.0f;
  if (lane == 0) scales[grp] = s2;
  const double s2d = static_cast<double>(s2);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const long long b = grp * 256 + lane * 8 + j;
    if (b < nb) {
      double q = rint(d[j] / s2d);
      q = fmin(127.0, fmax(-127.0, q));
      q8[b] = static_cast<int8_t>(q);
    }
  }
}

// Standalone dequantiser: one thread per code byte (2 elements).
__global__ void nf4_dequant_kernel(const uint8_t* __restrict__ codes, const int8_t* __restrict__ q8,
                                   const float* __restrict__ scales, const float* __restrict__ mean, long long n,
                                   uint16_t* __restrict__ out, const LUT16 lut) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long e = 2 * i;
  if (e >= n) return;
  const long long blk = e >> 6;
  const float mh = __fadd_rn(__fmul_rn(static_cast<float>(q8[blk]), scales[blk >> 8]), *mean);
  const uint8_t c = codes[i];
  const __nv_bfloat16 a = __float2bfloat16_rn(__fmul_rn(lut.v[c & 15], mh));
  out[e] = *reinterpret_cast<const uint16_t*>(&a);
  if (e + 1 < n) {
    const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(lut.v[c >> 4], mh));
    out[e + 1] = *reinterpret_cast<const uint16_t*>(&b);
  }
}

}  // namespace

cudaError_t nf4_quantize_launch(const float* w, long long n, uint8_t* codes, int8_t* q8, float* scales, float* mean,
                                float* absmax_scratch, const LUT16& lut, cudaStream_t st) {
  if (n <= 0) return cudaErrorInvalidValue;
  const long long nb = (n + 63) / 64;
  const long long ng = (nb + 255) / 256;
  nf4_block_codes_kernel<<<static_cast<unsigned>((nb * 32 + 255) / 256), 256, 0, st>>>(w, n, nb, codes, absmax_scratch,
                                                                                         lut);
  nf4_mean_kernel<<<1, 1024, 0, st>>>(absmax_scratch, nb, mean);
  nf4_dq_kernel<<<static_cast<unsigned>((ng * 32 + 255) / 256), 256, 0, st>>>(absmax_scratch, nb, mean, q8, scales);
  g_kernel_launches += 3;
  return cudaGetLastError();
}

cudaError_t nf4_dequant_launch(const uint8_t* codes, const int8_t* q8, const float* scales, const float* mean,
                               long long n, uint16_t* out, const LUT16& lut, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const long long nbytes = (n + 1) / 2;
  nf4_dequant_kernel<<<static_cast<unsigned>((nbytes + 255) / 256), 256, 0, st>>>(codes, q8, scales, mean, n, out, lut);
  ++g_kernel_launches;
  return cudaGetLastError();
}

}  // namespace soup

// ---------------------------------------------------------------- allocation-free variant
// Absmax scratch for soup_nf4_quantize_static: one block of 64 elements per entry, so the
// 1 Mi entries (4 MiB) cover tensors of up to 64 Mi elements.  Lives for the process.
namespace soup {
namespace {
constexpr long long kStaticBlocks = 1ll << 20;
static_assert(kStaticBlocks * 64 == SOUP_NF4_STATIC_MAX_ELEMS, "limit in soup.h");
static __device__ __align__(256) float g_static_absmax[kStaticBlocks];

// Device address of g_static_absmax per device ordinal (host code may not use the symbol's
// name as a pointer: that is a host-side stand-in, not a device address).  The address is
// looked up again on every call made outside stream capture, so a context recreated after
// cudaDeviceReset (which reloads the module, possibly elsewhere) is picked up; a call made
// while `stream` is capturing uses the address found by the last call outside capture.
std::mutex g_static_mu;
float* g_static_ptr[64] = {};

soup_status static_scratch(cudaStream_t stream, float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SOUP_ERR_CUDA;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return SOUP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_absmax) != cudaSuccess || !p) {
      g_static_ptr[dev] = nullptr;
      return SOUP_ERR_CUDA;
    }
    g_static_ptr[dev] = static_cast<float*>(p);
  } else if (!g_static_ptr[dev]) {
    return SOUP_ERR_STATE;  // no call outside capture has looked the address up on this device
  }
  *out = g_static_ptr[dev];
  return SOUP_OK;
}
}  // namespace
}  // namespace soup

const soup::LUT16& soup_codebook_lut();

extern "C" soup_status soup_nf4_quantize_static(const float* w, long long n, uint8_t* codes, int8_t* q8,
                                                float* scales, float* mean, void* stream) {
  if (!w || n <= 0 || !codes || !q8 || !scales || !mean) return SOUP_ERR_INVALID_ARG;
  if (n > SOUP_NF4_STATIC_MAX_ELEMS) return SOUP_ERR_INVALID_ARG;
  float* scratch = nullptr;
  const soup_status s = soup::static_scratch(static_cast<cudaStream_t>(stream), &scratch);
  if (s != SOUP_OK) return s;
  const cudaError_t e = soup::nf4_quantize_launch(w, n, codes, q8, scales, mean, scratch, soup_codebook_lut(),
                                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SOUP_OK : SOUP_ERR_CUDA;
}
