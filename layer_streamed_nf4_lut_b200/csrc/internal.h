// Internal declarations shared by the libsoup translation units (not part of the C-ABI).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

#include <atomic>

namespace soup {

// ----------------------------------------------------------------- NF4 tensor views
// One NF4 tensor W[rows, cols] (row-major flattened, blocks of 64, DQ groups of 256 blocks)
// stacked at row `row_begin` of a group that a GEMM sees as one matrix.
struct NF4Seg {
  const uint8_t* codes;  // packed codes, element 2i in the low nibble of byte i
  const int8_t* q8;      // double-quantised absmax, one per 64-element block
  const float* scales;   // fp32 scale per group of 256 blocks
  const float* mean;     // fp32 per-tensor mean of the absmax (device scalar)
  int row_begin;
  int rows;
};
struct NF4Group {
  NF4Seg seg[3];
  int nseg;
  int cols;        // in-dimension shared by the stacked tensors (multiple of 8)
  int total_rows;  // sum of rows
};

// ----------------------------------------------------------------- GEMM operands
// Element (r, k) of an operand that the GEMM reads as "row r, reduction index k".
enum OpKind : int {
  OP_BF16_K = 0,   // bf16 at ptr[r*ld + k]
  OP_BF16_MN = 1,  // bf16 at ptr[k*ld + r]
  OP_F32_K = 2,    // fp32 at ptr[r*ld + k], times `scale`, rounded to bf16
  OP_F32_MN = 3,   // fp32 at ptr[k*ld + r], times `scale`, rounded to bf16
  OP_NF4_K = 4,    // W[r, k] of the GEMM's NF4 group (forward: y = x W^T)
  OP_NF4_MN = 5,   // W[k, r] of the GEMM's NF4 group (backward: dx = dy W)
};

struct Operand {
  int kind;
  const void* ptr;
  long long ld;
  float scale;
  int row_lo, row_hi;  // rows outside [row_lo, row_hi) read as zero (block-diagonal LoRA)
};

struct GemmSeg {
  int K;
  Operand A;  // rows = GEMM M
  Operand B;  // rows = GEMM N
};

constexpr int GEMM_MAX_SEG = 5;
constexpr int GEMM_COUNTERS = 16384;  // split-K tile counters per workspace

struct GemmParams {
  // filled by gemm_launch:
  CUtensorMap tmapA[GEMM_MAX_SEG];  // TMA descriptors of bf16 A operands
  CUtensorMap tmapB[GEMM_MAX_SEG];  // TMA descriptors of bf16 B operands
  CUtensorMap tmapCodes[3];         // TMA descriptors of each NF4 tensor's packed codes (raw staging)
  CUtensorMap tmapQ8[3];            // ... and of its q8 absmax
  int a_mode[GEMM_MAX_SEG];         // 0: producer warps load A; 1: TMA, K-major; 2: TMA, MN-major
  int b_mode[GEMM_MAX_SEG];         // same for B (bf16 operands only)
  int b_row0[GEMM_MAX_SEG];         // first operand row of the B descriptor (block-diagonal windows)
  int raw_tma;                      // 1: the NF4 segment's codes / absmax arrive by TMA
  int bn;                           // output tile width
  int M, N;
  int nseg;
  GemmSeg seg[GEMM_MAX_SEG];
  NF4Group nf4;
  float lut[16];
  // epilogue: out[r, c] (or out[c, r] when out_trans) = alpha * acc (+ residual) (+ old out)
  void* out;
  long long ldo;
  int out_f32;
  int out_trans;
  float alpha;
  int accumulate;
  const void* residual;  // bf16, same layout as out (not with out_trans)
  long long ldr;
  // RoPE in the epilogue (the q | k columns of a q|k|v projection): output columns [0, rope_cols)
  // are heads of rope_d columns; each pair (i, i + rope_d/2) of a head is rotated by the angle of
  // the row's position, read from [positions, rope_d/2] cos / sin tables, on the fp32 result
  // before it is rounded.  Position of row r: r mod rope_S, less rope_rl for the last rope_rl
  // rows of each block (the rejected response of a shared-prefix pair block).  rope_cols = 0: off.
  const float* rope_cos;
  const float* rope_sin;
  int rope_cols, rope_d, rope_S, rope_rl;
  int* err;
  // split-K: when workspace and tile_counters are given, gemm_launch may split the K loop over
  // `splits` CTAs that write fp32 partial tiles to the workspace; they are summed in split order
  // by the last CTA of a tile to finish (counted in tile_counters, which it resets to 0) or by
  // a second kernel
  float* workspace;
  size_t ws_bytes;
  int* tile_counters;  // n_counters ints, zero between launches
  int n_counters;
  int splits;          // set by gemm_launch
  int fused_reduce;    // set by gemm_launch: 1 = the tile's last split sums the partials,
                       // 0 = a second kernel sums them (many splits: the sum runs wide)
  // stream-K (set by gemm_launch): sk_ctas > 0 spreads the sk_tiles x sk_nkt k-blocks of the
  // output tiles (M-tiles fastest, sk_tiles_m of them per N-tile) evenly over sk_ctas CTAs;
  // partial tiles go through the workspace (two slots per CTA) and the tile counters
  int sk_ctas;
  int sk_tiles;
  int sk_tiles_m;
  int sk_nkt;
};

// TMA descriptor of a 2D bf16 array (inner x outer elements, rows row_bytes apart), box
// box_inner x box_outer, 128-byte swizzle (box_inner * 2 must be 128), zero fill out of bounds.
// Cached by its arguments.  False if the driver refuses it (alignment, sizes).
bool tma_encode_bf16_sw128(CUtensorMap* map, const void* ptr, unsigned long long inner, unsigned long long outer,
                           unsigned long long row_bytes, unsigned box_inner, unsigned box_outer);

// The same array seen as 64-element column blocks ("planes", 128 B apart) of `rows` rows: a
// 3D map (64, rows, planes) whose box (64, box_rows, box_planes) lands in shared memory as
// box_planes consecutive [box_rows x 128 B] swizzled tiles, i.e. box_planes 64-wide column
// blocks of a row range in one copy.
bool tma_encode_bf16_sw128_planes(CUtensorMap* map, const void* ptr, unsigned long long rows, unsigned long long planes,
                                  unsigned long long row_bytes, unsigned box_rows, unsigned box_planes);

// Launch C = sum_seg A_seg B_seg^T on the tcgen05 tensor cores. Returns cudaError_t of launch.
cudaError_t gemm_launch(const GemmParams& p, cudaStream_t st);

// How gemm_launch schedules a GEMM (host only, no CUDA calls): tile (mt 128-row halves x bn
// columns), split-K count, or the stream-K partition over `sms` CTAs.
struct GemmPlan {
  int mt, bn, splits, fused_reduce;
  int sk_ctas, sk_tiles, sk_tiles_m, sk_nkt;
};
GemmPlan gemm_plan(const GemmParams& p, int sms, bool stream_k_allowed);

// ---- stream-K partition (host and device).  The k-blocks of `tiles` output tiles, nkt per
// tile, flattened tile by tile, are cut into `ctas` ranges: CTA c owns [bound(c), bound(c+1)).
__host__ __device__ inline long long sk_bound(long long tiles, int nkt, int ctas, int c) {
  return tiles * nkt * c / ctas;
}
// the CTA whose range holds flattened k-block x
__host__ __device__ inline int sk_owner(long long tiles, int nkt, int ctas, long long x) {
  const long long W = tiles * nkt;
  int c = static_cast<int>(x * ctas / W);
  while (c + 1 < ctas && sk_bound(tiles, nkt, ctas, c + 1) <= x) ++c;
  while (c > 0 && sk_bound(tiles, nkt, ctas, c) > x) --c;
  return c;
}
// pieces of CTA c: its range cut at tile boundaries (piece pc lies in tile first_tile + pc)
__host__ __device__ inline int sk_piece_count(long long tiles, int nkt, int ctas, int c) {
  const long long lo = sk_bound(tiles, nkt, ctas, c), hi = sk_bound(tiles, nkt, ctas, c + 1);
  return hi <= lo ? 0 : static_cast<int>((hi - 1) / nkt - lo / nkt + 1);
}
__host__ __device__ inline void sk_piece(long long tiles, int nkt, int ctas, int c, int pc, int* tile, int* kb_lo,
                                         int* kb_hi) {
  const long long lo = sk_bound(tiles, nkt, ctas, c), hi = sk_bound(tiles, nkt, ctas, c + 1);
  const long long t = lo / nkt + pc, t0 = t * nkt;
  *tile = static_cast<int>(t);
  *kb_lo = static_cast<int>((lo > t0 ? lo : t0) - t0);
  *kb_hi = static_cast<int>((hi < t0 + nkt ? hi : t0 + nkt) - t0);
}
// workspace slot of a partial piece: 2c for CTA c's first piece, 2c + 1 for its last (a
// partial tile is only ever cut at the two ends of a range)
__host__ __device__ inline int sk_slot(int c, int pc) { return 2 * c + (pc == 0 ? 0 : 1); }
// share k (in k order) of a tile cut between CTAs: its CTA and slot; the count is
// sk_owner(last k-block) - sk_owner(first) + 1
__host__ __device__ inline void sk_share(long long tiles, int nkt, int ctas, int tile, int k, int* cta, int* slot) {
  const long long x0 = static_cast<long long>(tile) * nkt;
  const int c = sk_owner(tiles, nkt, ctas, x0) + k;
  *cta = c;
  *slot = 2 * c + ((k == 0 && sk_bound(tiles, nkt, ctas, c) < x0) ? 1 : 0);
}

// ----------------------------------------------------------------- NF4 quantiser / dequant
struct LUT16 {
  float v[16];
};
cudaError_t nf4_quantize_launch(const float* w, long long n, uint8_t* codes, int8_t* q8, float* scales, float* mean,
                                float* absmax_scratch, const LUT16& lut, cudaStream_t st);
// Host quantiser (host_quant.cu): the same bytes as nf4_quantize_launch, from host memory,
// on `threads` host threads (<= 0: all hardware threads).  Returns a soup_status.
int host_nf4_quantize(const float* w, long long n, uint8_t* codes, int8_t* q8, float* scales, float* mean,
                      int threads);
cudaError_t nf4_dequant_launch(const uint8_t* codes, const int8_t* q8, const float* scales, const float* mean,
                               long long n, uint16_t* out, const LUT16& lut, cudaStream_t st);

// ----------------------------------------------------------------- attention
struct AttnShape {
  int B, S, hq, hkv, d;
  long long ld_qkv;  // row stride (elements) of the [T, (hq+2hkv)d] qkv buffer
  // Shared-prefix pair layout (pl > 0): each of the B blocks of S = pl + 2 rl rows holds one
  // preference pair as [prefix (pl) | chosen response (rl) | rejected response (rl)]; the
  // rejected rows sit at positions pl.. and see the prefix and their own earlier rows, never
  // the chosen ones.  pl = 0: plain causal rows.
  int pl, rl;
  // RoPE cos / sin tables [positions, d/2] (the forward rotation is applied in the q|k|v GEMM):
  // the backward rotates dQ and dK back by the same angles before writing them; NULL: no rotation
  const float* rope_cos;
  const float* rope_sin;
};
// Forward (attention.cu, tcgen05): o [T, hq d] bf16, lse [B, hq, S] fp32 (natural log); err: the
// device error word (a bounded in-kernel wait that ran out sets it).
cudaError_t attn_fwd_launch(const AttnShape& s, const uint16_t* qkv, uint16_t* o, float* lse, int* err,
                            cudaStream_t st);
// Backward: delta [T, hq] fp32 scratch, dQ / dK / dV written into dqkv (same layout as qkv).  ws:
// fp32 scratch (16-byte aligned) for per-head-slice dK / dV partials when the kv grid alone
// cannot fill the GPU; NULL / too small: no head slices.
cudaError_t attn_bwd_launch(const AttnShape& s, const uint16_t* qkv, const uint16_t* o, const uint16_t* dout,
                            const float* lse, float* delta, uint16_t* dqkv, float* ws, size_t ws_bytes, int* err,
                            cudaStream_t st);
// delta[t, h] = sum_d dO * O, and the slice-order sum of per-head-slice dK / dV partials
cudaError_t attn_delta_launch(const uint16_t* o, const uint16_t* dout, int T, int hq, int d, float* delta,
                              cudaStream_t st);
cudaError_t attn_dkdv_sum_launch(const AttnShape& s, int hsplit, const float* part, uint16_t* dqkv, cudaStream_t st);

// ----------------------------------------------------------------- elementwise / row ops
cudaError_t embed_launch(const int32_t* ids, const uint16_t* table, int T, int h, int V, uint16_t* out, int* err,
                         cudaStream_t st);
cudaError_t rmsnorm_fwd_launch(const uint16_t* x, const uint16_t* gamma, int T, int h, float eps, uint16_t* y,
                               float* rstd, cudaStream_t st);
cudaError_t rmsnorm_bwd_launch(const uint16_t* dy, const uint16_t* x, const float* rstd, const uint16_t* gamma,
                               const uint16_t* dres, int T, int h, uint16_t* dx, cudaStream_t st);
cudaError_t swiglu_fwd_launch(const uint16_t* gu, int T, int I, uint16_t* m, cudaStream_t st);
cudaError_t swiglu_bwd_launch(const uint16_t* dm, const uint16_t* gu, int T, int I, uint16_t* dgu, cudaStream_t st);
cudaError_t ce_rows_launch(const float* logits, int T, int V, const int32_t* ids, int B, int S, const uint8_t* mask,
                           int resp_start, float* lse, float* tgt_logit, int* err, cudaStream_t st);
cudaError_t sft_finish_launch(const float* lse, const float* tgt, const int32_t* ids, int B, int S, const uint8_t* mask,
                              float* loss_out, float* row_weight, cudaStream_t st);
cudaError_t dpo_finish_launch(const float* lse, const float* tgt, int B, int S, int resp_start, int n_pairs, float beta,
                              const float* ref_logp, float* pi_out, float* loss_out, float* row_weight,
                              cudaStream_t st);
enum PrefKind { PREF_KTO = 2, PREF_ORPO = 3, PREF_SIMPO = 4 };  // values of soup_loss
cudaError_t pref_finish_launch(int kind, const float* lse, const float* tgt, int B, int S, int resp_start,
                               const float* ref_logp, const uint8_t* labels, float beta, float gamma, float lam_or,
                               float lam_d, float lam_u, float* pi_out, float* loss_out, float* row_weight,
                               cudaStream_t st);
// Loss closed forms on precomputed per-sequence sums, writing seq_w = -dL/dpi per sequence.
cudaError_t dpo_loss_seqw_launch(const float* pi, const float* ref_logp, int n_pairs, float beta, float* loss_out,
                                 float* seq_w, cudaStream_t st);
cudaError_t pref_loss_seqw_launch(int kind, const float* pi, const float* ref_logp, const uint8_t* labels, int B,
                                  int n_resp, float beta, float gamma, float lam_or, float lam_d, float lam_u,
                                  float* loss_out, float* seq_w, cudaStream_t st);
// Shared-prefix pair blocks: packing, two-target rows, per-pair log-prob sums, row weights.
cudaError_t pair_pack_launch(const int32_t* ids, int P, int S, int pl, int V, int32_t* pids, int32_t* tgt1,
                             int32_t* tgt2, int* err, cudaStream_t st);
cudaError_t ce_rows_t_launch(const float* logits, int T, int V, const int32_t* tgt1, const int32_t* tgt2, float* lse,
                             float* rt1, float* rt2, cudaStream_t st);
cudaError_t pair_logp_launch(const float* lse, const float* rt1, const float* rt2, int P, int pl, int rl, float* out,
                             cudaStream_t st);
cudaError_t pair_rowweight_launch(const float* seq_w, int P, int pl, int rl, float* w1, float* w2, cudaStream_t st);
cudaError_t ce_grad_t_launch(const float* logits, const float* lse, const int32_t* tgt1, const float* w1,
                             const int32_t* tgt2, const float* w2, int T, int V, uint16_t* dlogits, cudaStream_t st);
cudaError_t seq_logp_launch(const float* lse, const float* tgt, int B, int S, int resp_start, float* out,
                            cudaStream_t st);
cudaError_t ce_grad_launch(const float* logits, const float* lse, const int32_t* ids, const float* row_weight, int B,
                           int S, int V, uint16_t* dlogits, cudaStream_t st);
// AdamW on fp32 parameters; also writes their bf16 copy `pb` (may be null).
cudaError_t adamw_launch(float* p, const float* g, float* m, float* v, uint16_t* pb, long long n, float lr, float b1,
                         float b2, float eps, float wd, int t, cudaStream_t st);
// The same update with lr and the bias corrections read from device memory (hp[0] = lr,
// hp[1] = 1/(1-b1^t), hp[2] = 1/(1-b2^t)), so that a captured graph applies each step's values.
cudaError_t adamw_hp_launch(float* p, const float* g, float* m, float* v, uint16_t* pb, long long n, float b1,
                            float b2, float eps, float wd, const float* hp, cudaStream_t st);
// 1/(1-b1^t) and 1/(1-b2^t) as the update uses them
void adamw_bias_corrections(float b1, float b2, int t, float* bc1, float* bc2);
cudaError_t busy_wait_launch(long long cycles, cudaStream_t st);  // profiling aid, not counted as a launch
cudaError_t null_launch(cudaStream_t st);
// one thread waits on a barrier nothing arrives on, limit_ns ns, then sets *err (timeout)
cudaError_t bounded_wait_selftest_launch(int* err, unsigned long long limit_ns, cudaStream_t st);                           // profiling aid, not counted as a launch
cudaError_t f32_to_bf16_launch(const float* x, uint16_t* y, long long n, cudaStream_t st);
cudaError_t fill_zero_launch(void* p, size_t bytes, cudaStream_t st);

// ----------------------------------------------------------------- launch accounting
// Number of kernels this library has launched (process-wide, monotonically increasing).
extern std::atomic<long long> g_kernel_launches;

}  // namespace soup
