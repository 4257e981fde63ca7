/*
 * libsoup — layer-streamed NF4 + LoRA training step on one B200 (sm_100a).
 *
 * The method (as described on the pages about the open-source "Soup" trainer):
 *   - the frozen base model is kept outside GPU memory and fed to the GPU one decoder
 *     layer at a time: load the layer, compute its activation, drop it, go to the next
 *     (rug.gal radar "Soup ... layer streaming", section "En detalle"; imasters "Como cabe um
 *     8B em 4 GB");
 *   - the base is NF4 4-bit quantised; only the LoRA adapters and the current batch stay on
 *     the GPU (same sections; soup.yaml example with `stream_layers: true`, `quantization: 4bit`);
 *   - streamed and resident runs give the same result bit for bit, because streaming only
 *     reorders when data reaches the GPU (rug.gal "En detalle"; guillermodelpino "El streaming
 *     de capas, que es el truco de la casa"; imasters "Do SFT para os métodos de preferência");
 *   - DPO obtains its reference log-probs by re-streaming the same base with the LoRA adapters
 *     switched off: one set of weights, one stream (rug.gal "En detalle"; imasters "Do SFT ...").
 *
 * Conventions for every entry point:
 *   - every call returns soup_status: SOUP_OK (0) or a negative code; no exception crosses
 *     the boundary; out-parameters are written only on success;
 *   - soup_last_error(model) returns a message owned by the model, valid until the next call;
 *   - "device" pointers are CUDA device addresses on the model's device, "host" pointers are
 *     CPU addresses; bf16 tensors are passed as their 16-bit patterns;
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream); calls
 *     enqueue work on it and return without synchronising unless stated; the layer streamer
 *     uses one internal copy stream fenced with CUDA events;
 *   - a model is not thread-safe: one host thread at a time per model;
 *   - shapes: hidden, head_dim*heads, intermediate and lora_r must be multiples of 8;
 *     head_dim must be 64 or 128; vocab a multiple of 4.  Other shapes -> SOUP_ERR_UNSUPPORTED.
 */
#ifndef SOUP_H_
#define SOUP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t soup_status;
#define SOUP_OK 0
#define SOUP_ERR_INVALID_ARG (-1)  /* null pointer, out-of-range index, bad size */
#define SOUP_ERR_STATE (-2)        /* wrong call order (e.g. backward without forward, missing weights) */
#define SOUP_ERR_OOM (-3)          /* host pinned or device allocation failed */
#define SOUP_ERR_CUDA (-4)         /* a CUDA runtime call failed */
#define SOUP_ERR_TIMEOUT (-5)      /* a bounded wait (host event or in-kernel barrier) ran out */
#define SOUP_ERR_DEVICE_CHECK (-6) /* a kernel's bounds check fired (e.g. token id >= vocab) */
#define SOUP_ERR_UNSUPPORTED (-7)  /* shape outside what the kernels implement */
#define SOUP_ERR_IO (-8)           /* the file-backed layer stack failed to read or write */

typedef struct soup_model soup_model;

enum { SOUP_RESIDENT = 0, SOUP_STREAMED = 1 };
/* Where the NF4 layer stack lives on the host side (the pages' stream_source). */
enum { SOUP_SOURCE_RAM = 0, SOUP_SOURCE_FILE = 1, SOUP_SOURCE_AUTO = 2 };
enum { SOUP_PROJ_Q = 0, SOUP_PROJ_K, SOUP_PROJ_V, SOUP_PROJ_O, SOUP_PROJ_GATE, SOUP_PROJ_UP, SOUP_PROJ_DOWN, SOUP_N_PROJ };
typedef enum {
  SOUP_LOSS_SFT = 0,
  SOUP_LOSS_DPO = 1,
  SOUP_LOSS_KTO = 2,   /* reference from the LoRA-off re-stream, like DPO */
  SOUP_LOSS_ORPO = 3,  /* reference-free */
  SOUP_LOSS_SIMPO = 4  /* reference-free */
} soup_loss;

/* Model shape and run options.  Decoder layer = pre-norm Llama block (RMSNorm, GQA attention
 * with rotate-half RoPE, SwiGLU MLP), LoRA on all seven projections with scale alpha/r. */
typedef struct soup_model_config {
  int n_layers, hidden, n_heads, n_kv_heads, head_dim, intermediate, vocab;
  float rms_eps, rope_theta;
  int lora_r;
  float lora_alpha;
  int mode;            /* SOUP_RESIDENT (every layer on the device) or SOUP_STREAMED */
  int n_layer_buffers; /* streamed: device layer buffers, >= 2 (the resident-layer budget) */
  int max_tokens;      /* largest B*S any call will use (sizes the activation storage) */
  int device;          /* CUDA device ordinal */
  int stream_source;   /* SOUP_SOURCE_RAM (0): page-locked host RAM, one blob per layer.
                          SOUP_SOURCE_FILE: one file at stack_path (created / truncated by
                          soup_model_create), layer i at i * stride (blob bytes rounded up to
                          4096); a reader thread fills n_layer_buffers page-locked staging
                          slots ahead of the copies.  SOUP_SOURCE_AUTO: RAM if the stack fits in
                          half the host's free physical memory, else FILE (needs stack_path). */
  const char* stack_path; /* FILE / AUTO: path of the layer stack file; may be NULL for RAM */
} soup_model_config;

/* Optional device allocator (e.g. routed to PyTorch's caching allocator).  alloc returns
 * NULL on failure.  With a NULL soup_allocator the library calls cudaMalloc / cudaFree. */
typedef struct soup_allocator {
  void* (*alloc)(size_t bytes, void* user);
  void (*free)(void* ptr, void* user);
  void* user;
} soup_allocator;

/* Per-model counters since creation (or the last soup_reset_stats). */
typedef struct soup_stats {
  long long layer_loads;      /* host->device layer copies issued by the streamer */
  long long bytes_h2d;        /* bytes of those copies */
  long long layer_reuses;     /* layer requests served by an already-resident buffer */
  long long kernel_launches;  /* kernels this model's calls launched */
  long long device_bytes;     /* device bytes the model holds (weights buffers, activations, scratch) */
  long long pinned_bytes;     /* page-locked host bytes holding the NF4 layer stack */
  long long steps;            /* completed soup_step calls */
  long long file_bytes_read;  /* file source: bytes read from the stack file into staging */
  double file_read_ms;        /* file source: wall time of those reads (reader thread) */
  int stream_source;          /* the source in use: SOUP_SOURCE_RAM or SOUP_SOURCE_FILE */
} soup_stats;

/* One training batch.  Token ids are [B, S] row-major int32.
 * SFT: row t = (b, s) predicts ids[b, s+1]; targets are positions j >= 1 of each sequence,
 *      optionally filtered by loss_mask[b, j] != 0 (uint8 [B, S]); loss = token mean.
 * Preference losses act on per-sequence sums of target log-probs over the response, targets
 * j >= max(prefix_len, 1): pi with LoRA on (fp32 sums), ref the same with LoRA off; n = S -
 * max(prefix_len, 1) response targets per row; sigma = logistic function.
 * DPO (Rafailov et al. 2023): B = 2 * n_pairs; rows 2p (chosen) and 2p+1 (rejected);
 *      loss = -mean_p log sigma(beta [(pi_c - ref_c) - (pi_r - ref_r)]).
 * SimPO (Meng et al. 2024): pairs as DPO, no reference; a = pi / n;
 *      loss = -mean_p log sigma(beta (a_c - a_r) - gamma).
 * ORPO (Hong et al. 2024): pairs as DPO, no reference; odds(a) = e^a / (1 - e^a);
 *      loss = mean_p [-a_c - lambda_or log sigma(log odds(a_c) - log odds(a_r))].
 * KTO (Ethayarajh et al. 2024): B unpaired rows, labels[b] != 0 desirable; r = pi - ref;
 *      z0 = max(0, mean_b r_b) with no gradient through it; v_b = lambda_d sigma(beta (r_b -
 *      z0)) if desirable, lambda_u sigma(beta (z0 - r_b)) if not; loss = mean_b (lambda_b - v_b).
 * ids_on_host != 0: ids / loss_mask / labels are host pointers; the library copies them to
 *      the device on `stream` inside the call (pageable or pinned memory both accepted). */
typedef struct soup_batch {
  const int32_t* ids;
  const uint8_t* loss_mask; /* may be NULL */
  int B, S;
  int ids_on_host;
  int n_pairs, prefix_len;
  float beta;
  float lr;            /* AdamW learning rate (betas 0.9/0.999, eps 1e-8, weight decay 0) */
  int apply_optimizer; /* 0: leave gradients in the grad buffer, do not update */
  int dpo_shared_load; /* DPO and KTO.  0: the reference forward re-streams the whole stack
                          with LoRA off, then the policy forward streams it again (3L-2 loads
                          from a cold streamer).  1: each layer is loaded once and runs the
                          LoRA-off and the LoRA-on forward back to back (2L-2 loads); same bits. */
  const uint8_t* labels; /* KTO: uint8 [B], desirable != 0 (same memory space as ids) */
  float gamma;           /* SimPO target margin */
  float lambda_or;       /* ORPO weight of the odds-ratio term */
  float lambda_d, lambda_u; /* KTO weights of desirable / undesirable rows */
  int share_prefix;      /* DPO, SimPO, ORPO: 1 = each pair's shared prefix (ids[2p][:prefix_len] ==
                            ids[2p+1][:prefix_len], the caller's promise) runs through the layers
                            once: the pair becomes one block [prefix | chosen | rejected] in which
                            the rejected response attends to the prefix and to itself.  Applies
                            when prefix_len and S - prefix_len are multiples of 64 (else the plain
                            layout runs); the same loss and gradients up to rounding order. */
} soup_batch;

/* ---- lifecycle -------------------------------------------------------------------------- */

/* Creates a model: validates cfg, computes the NF4 codebook, allocates the page-locked host
 * layer stack (n_layers blobs), the device layer buffers (n_layers resident, n_layer_buffers
 * streamed), activation storage for max_tokens and scratch.  Weights are loaded afterwards.
 * The host-side stack and the few device layer buffers are the pages' layer streaming: the
 * base lives in CPU RAM (or on disk, stream_source) and the GPU holds one layer at a time
 * plus the adapters (rug.gal radar "Soup ... layer streaming", "En detalle"; imasters "Como
 * cabe um 8B em 4 GB").  SOUP_ERR_UNSUPPORTED for shapes outside the kernels, SOUP_ERR_OOM
 * when an allocation (or the caller's allocator) fails; nothing is leaked on failure.
 * soup_model_destroy frees everything the model holds (NULL: SOUP_ERR_INVALID_ARG). */
soup_status soup_model_create(const soup_model_config* cfg, const soup_allocator* alloc, soup_model** out);
soup_status soup_model_destroy(soup_model* model);

/* Bytes of one layer's NF4 blob (7 projections: codes, q8 absmax, fp32 group scales, fp32
 * mean; then the two bf16 RMSNorm gains), each part 256-byte aligned: the unit the streamer
 * moves (rug.gal "En detalle": one decoder layer is loaded, used and dropped). */
soup_status soup_layer_blob_bytes(const soup_model_config* cfg, size_t* bytes);

/* Quantises one layer on the device into the model's host layer stack (NF4, the pages'
 * `quantization: 4bit`: guillermodelpino soup.yaml example; rug.gal "En detalle").
 * w[p]: device fp32 [out_p, in_p] row-major for p = q,k,v,o,gate,up,down; gammas: device bf16
 * [hidden].  Runs the NF4 + double-quant kernels, then copies the blob to page-locked host
 * memory (synchronises `stream`).  In resident mode the blob is also kept on the device. */
soup_status soup_model_quantize_layer(soup_model* model, int layer, const float* const w[7],
                                      const uint16_t* gamma_attn, const uint16_t* gamma_mlp, void* stream);
/* Loads one layer from float32 weights in HOST memory: the library quantises them on the host
 * (all hardware threads; the same bytes as soup_model_quantize_layer and soup_nf4_quantize_host)
 * straight into its page-locked layer stack (or the stack file), so a base that never fits on
 * the GPU in float32 never has to be there (rug.gal radar "Soup ... layer streaming", "En
 * detalle": the base stays in CPU RAM and reaches the GPU one quantised layer at a time).
 * w[p]: host fp32 [out_p, in_p] row-major for p = q,k,v,o,gate,up,down; gammas: host bf16
 * [hidden].  Synchronous: waits for the streamer's copy stream first (it may be reading an older
 * blob of this layer), returns when the blob is stored; in resident mode the blob is also
 * copied to the layer's device buffer.  SOUP_ERR_INVALID_ARG for a NULL pointer or a bad layer
 * index; SOUP_ERR_IO when the stack file cannot be written. */
soup_status soup_model_load_layer(soup_model* model, int layer, const float* const w[7], const uint16_t* gamma_attn,
                                  const uint16_t* gamma_mlp);
/* Loads / reads back a pre-quantised blob (host memory, soup_layer_blob_bytes bytes) into or
 * out of the model's host layer stack (the CPU-RAM or disk copy the pages stream from: rug.gal
 * "En detalle"; imasters "Como cabe um 8B em 4 GB").  Synchronous.  SOUP_ERR_INVALID_ARG for
 * a bad layer index or a size other than soup_layer_blob_bytes; SOUP_ERR_IO on a file error. */
soup_status soup_model_load_layer_nf4(soup_model* model, int layer, const void* blob, size_t bytes);
soup_status soup_model_read_layer_nf4(soup_model* model, int layer, void* blob, size_t bytes);
/* Byte offset and size of a part of projection p inside a layer blob; part 0 = codes, 1 = q8
 * absmax, 2 = group scales, 3 = mean; p = 7 gives the attention gain, p = 8 the MLP gain. */
soup_status soup_layer_blob_part(const soup_model_config* cfg, int proj, int part, size_t* offset, size_t* bytes);

/* Frozen head weights (device, bf16, caller-owned, kept by pointer): embedding [vocab, hidden],
 * final RMSNorm gain [hidden], lm_head [vocab, hidden].  They stay resident: the pages stream
 * the decoder layers only (rug.gal "En detalle"). */
soup_status soup_model_set_head(soup_model* model, const void* embed, const void* final_gamma, const void* lm_head);

/* LoRA storage (the trained adapters, which stay in VRAM: rug.gal "En detalle"; guillermodelpino
 * soup.yaml example, r and alpha): four caller-owned device fp32 buffers of soup_lora_numel elements each
 * (parameters, gradients, AdamW first and second moments; moments start at zero).  Layout:
 * layer-major; inside a layer A_q, A_k, A_v, A_o, A_gate, A_up, A_down (each [r, in]) then
 * B_q, ..., B_down (each [out, r]), row-major.  soup_lora_offset gives each tensor's place. */
soup_status soup_lora_numel(const soup_model_config* cfg, size_t* numel);
soup_status soup_lora_offset(const soup_model_config* cfg, int layer, int proj, int which_b, size_t* offset,
                             int* rows, int* cols);
soup_status soup_model_set_lora(soup_model* model, float* params, float* grads, float* adam_m, float* adam_v);
/* Sets the adapters of one projection: copies A [r, in] and B [out, r] (fp32, row-major, host
 * or device memory) into the parameter buffer given to soup_model_set_lora, at the place
 * soup_lora_offset names, and refreshes their bf16 copy; enqueued on `stream`.  The adapters
 * are the rank-r pair of each adapted projection (guillermodelpino soup.yaml example: r,
 * alpha; rug.gal "En detalle": only the adapter is trained).  SOUP_ERR_STATE before
 * soup_model_set_lora; SOUP_ERR_INVALID_ARG for a bad layer or projection index. */
soup_status soup_model_set_lora_proj(soup_model* model, int layer, int proj, const float* A, const float* B,
                                     void* stream);
/* The kernels read the LoRA parameters through a bf16 copy kept by the library (the values
 * the fp32 parameters round to), refreshed by soup_model_set_lora (synchronous) and by every
 * optimizer update the library performs.  A caller that changes the fp32 parameters itself
 * calls soup_model_refresh_lora (enqueued on `stream`) before the next forward. */
soup_status soup_model_refresh_lora(soup_model* model, void* stream);

/* LoRA on/off for the forward and backward calls that follow.  Off: the LoRA branch and its
 * gradients are skipped entirely (not multiplied by zero), which is the DPO reference model:
 * the same base stream with the adapters switched off (rug.gal "En detalle"; imasters "Do SFT
 * para os métodos de preferência").  Always SOUP_OK for a valid model. */
soup_status soup_set_lora_enabled(soup_model* model, int enabled);

/* Merged weight of one projection: out = bf16(W + (lora_alpha / lora_r) * B * A), device bf16
 * [out_features, in_features] row-major (the layout of the projection's NF4 tensor, q|k|v and
 * gate|up NOT stacked), 16-byte aligned, caller-owned.  W is the dequantised NF4 base, A and
 * B the projection's adapters (their bf16 values, as the training forward uses them); the
 * product accumulates in fp32 and the sum is rounded once to bf16.  This is the pages' merge
 * command, which fuses the trained adapter into the base (guillermodelpino page, the commands
 * of the full cycle; imasters page, "O que muda para quem constrói no Brasil").  The layer is
 * taken from the streamer like a forward does (a streamed model may load it).  Runs on
 * `stream`.  SOUP_ERR_STATE before set_lora or before the layer has weights;
 * SOUP_ERR_INVALID_ARG for a bad layer / proj index or a misaligned `out`. */
soup_status soup_model_merge_lora(soup_model* model, int layer, int proj, void* out, void* stream);

/* ---- layer-level calls ------------------------------------------------------------------- */

/* One decoder layer forward: x_out = layer(x_in), device bf16 [B*S, hidden].  Acquires the
 * layer from the streamer (or the resident copy), keeps the activations needed by
 * soup_layer_bwd inside the model (per layer), runs every kernel on `stream`.  The layer is
 * the Llama-3.1-8B decoder layer the pages stream one at a time (rug.gal lead and "En
 * detalle"; guillermodelpino "El streaming de capas, que es el truco de la casa"). */
soup_status soup_layer_fwd(soup_model* model, int layer, const void* x_in, void* x_out, int B, int S, void* stream);
/* Backward of the last soup_layer_fwd of this layer: dx = d(loss)/d(x_in) given
 * dy = d(loss)/d(x_out) (device bf16 [B*S, hidden]); ACCUMULATES the layer's LoRA gradients
 * into the grad buffer (callers zero it first); the base gets no gradient, it is frozen
 * (rug.gal "En detalle").  SOUP_ERR_STATE without a matching forward. */
soup_status soup_layer_bwd(soup_model* model, int layer, const void* dy, void* dx, int B, int S, void* stream);

/* ---- whole step -------------------------------------------------------------------------- */

/* One training step: embedding, streamed forward over all layers, head and loss, streamed
 * backward, LoRA gradients (zeroed first) and, if batch->apply_optimizer, the AdamW update
 * (each layer's LoRA slice is updated during the backward pass, as soon as its gradients are
 * complete, with the same arithmetic as soup_optimizer_step; a step that fails part-way may
 * leave some slices updated)
 * (the pages' SFT and preference training under layer streaming: rug.gal "En detalle";
 * imasters "Do SFT para os métodos de preferência"; guillermodelpino soup.yaml example, lr).
 * SFT streams 2L-2 layer loads from a cold streamer (the two top layers are reused at the
 * forward/backward turnaround); DPO and KTO add a full LoRA-off forward pass, 3L-2 loads
 * (2L-2 with dpo_shared_load); SimPO and ORPO stream like SFT.  Layers
 * still resident from the previous step are reused.  *loss_out (host) receives the loss
 * after the call synchronises `stream`. */
soup_status soup_step(soup_model* model, soup_loss loss, const soup_batch* batch, float* loss_out, void* stream);
/* AdamW update of all LoRA parameters from the grad buffer (step counter kept by the model);
 * the pages give only the learning rate (guillermodelpino soup.yaml example). */
soup_status soup_optimizer_step(soup_model* model, float lr, void* stream);
/* Per-sequence summed target log-probs of the last preference step (host fp32[B]): policy
 * and ref (ref is written by DPO and KTO only; it comes from the LoRA-off re-stream: rug.gal
 * "En detalle").  Copies the first n entries (1 <= n <= max_tokens, else SOUP_ERR_INVALID_ARG);
 * synchronous; entries no preference step has written are unspecified. */
soup_status soup_last_logps(soup_model* model, float* pi, float* ref, int n);

/* ---- single operations (each one kernel sequence, for tests and tools) ------------------- */

/* NF4 + double quantisation (the pages' `quantization: 4bit`: guillermodelpino soup.yaml
 * example; rug.gal "En detalle") of one device fp32 tensor of n elements (row-major flattened):
 * codes [ceil(n/2)] u8, q8 [ceil(n/64)] i8, scales [ceil(n/64/256)] f32, mean [1] f32, all
 * device; scratch: device f32 [ceil(n/64)] (absmax). */
soup_status soup_nf4_quantize(const float* w, long long n, uint8_t* codes, int8_t* q8, float* scales, float* mean,
                              float* scratch, void* stream);
/* Same quantiser, for callers that cannot call cudaMalloc (for example code running where
 * device allocation is not allowed, or whose device memory is all owned by another allocator)
 * and so cannot supply the absmax scratch buffer soup_nf4_quantize needs.  The paper has no
 * counterpart: this is a deployment convenience.  The scratch is a fixed array inside the
 * library (4 MiB of device memory on every GPU that loads the library, held until the
 * process exits), so n may be at most SOUP_NF4_STATIC_MAX_ELEMS (= 64 x 2^20 elements, every
 * 8B-shape projection); larger n returns SOUP_ERR_INVALID_ARG without launching anything.
 * The call allocates nothing.  Every call made outside stream capture looks up the array's
 * device address on the current device (so a context recreated by cudaDeviceReset is picked
 * up); a call made while `stream` is capturing reuses the address found by the last call
 * outside capture on that device, and returns SOUP_ERR_STATE if there was none: make the
 * first call on a device before any stream capture, and again after a cudaDeviceReset.  All
 * calls share the one array and it keeps the last call's contents; every entry a call reads
 * is written earlier in the same call, so nothing needs clearing, but calls whose kernels
 * overlap on the GPU (different streams, or different host threads) race on it: serialise
 * them.  Outputs and error behaviour are those of soup_nf4_quantize. */
#define SOUP_NF4_STATIC_MAX_ELEMS (64LL << 20)
soup_status soup_nf4_quantize_static(const float* w, long long n, uint8_t* codes, int8_t* q8, float* scales,
                                     float* mean, void* stream);
/* The same quantiser on the host: w and every output are HOST pointers (sizes as for
 * soup_nf4_quantize); runs on n_threads host threads (<= 0: all hardware threads) and returns
 * when done.  No GPU is needed.  The NF4 format of the pages' `quantization: 4bit`
 * (guillermodelpino soup.yaml example; rug.gal "En detalle"). */
soup_status soup_nf4_quantize_host(const float* w, long long n, uint8_t* codes, int8_t* q8, float* scales, float* mean,
                                   int n_threads);
/* Standalone NF4 -> bf16 dequantiser: out[i] = bf16_rn(c[code_i] * mhat(block(i))), the
 * decode every streamed GEMM applies to the 4-bit base (rug.gal "En detalle"). */
soup_status soup_nf4_dequantize(const uint8_t* codes, const int8_t* q8, const float* scales, const float* mean,
                                long long n, uint16_t* out, void* stream);
/* The streamed layer's projection on its own (rug.gal "En detalle": the 4-bit base is used
 * as it arrives): y[M, N] (bf16) = x[M, K] (bf16) . W^T + (residual) for one NF4 tensor W [N, K] (device
 * parts as produced by soup_nf4_quantize); transpose_w != 0 computes y[M, K] = x[M, N] . W.
 * The first call on a device allocates a 64 MiB workspace and tile counters for the
 * stream-K schedule, shared by later calls on that device: calls that overlap on the GPU
 * (different streams) must not be made. */
soup_status soup_nf4_matmul(const void* x, int M, int N, int K, const uint8_t* codes, const int8_t* q8,
                            const float* scales, const float* mean, int transpose_w, const void* residual, void* y,
                            void* stream);
/* ---- GEMM scheduling diagnostics (host only: no GPU needed, nothing launched) ----------- */
/* How the library schedules y[M, N] = x[M, K] . W^T for one operand W: nf4 != 0 for an NF4
 * weight (transposed != 0: the dX orientation, W read as [K, N]), else bf16; with the
 * library's own workspace (64 MiB, 16384 tile counters) on a device of `sms` SMs.  mt x bn is
 * the output tile (mt 128-row halves); splits > 1 splits K over that many CTAs per tile;
 * stream_k_ctas > 0 spreads stream_k_tiles x stream_k_kblocks k-blocks over that many CTAs
 * (see soup_gemm_stream_k_piece).  SOUP_ERR_INVALID_ARG for non-positive sizes or N, K not
 * multiples of 8. */
typedef struct soup_gemm_plan_info {
  int mt, bn, splits, fused_reduce;
  int stream_k_ctas, stream_k_tiles, stream_k_tiles_m, stream_k_kblocks;
} soup_gemm_plan_info;
soup_status soup_gemm_plan(int M, int N, int K, int nf4, int transposed, int sms, soup_gemm_plan_info* out);
/* The stream-K partition: pieces of CTA `cta` (at most max_pieces written; *n_pieces = count):
 * output tile, k-block range [kb_lo, kb_hi) within it, and the workspace slot a partial piece
 * stores its share in (-1 when the piece covers its whole tile). */
soup_status soup_gemm_stream_k_pieces(long long tiles, int kblocks_per_tile, int ctas, int cta, int max_pieces,
                                      int* tile, int* kb_lo, int* kb_hi, int* slot, int* n_pieces);
/* The shares of one tile, in k order (at most max_shares written; *n_shares = count): the CTA
 * that computes each and the workspace slot it is summed from.  A tile computed by one CTA
 * alone has one share with slot -1. */
soup_status soup_gemm_stream_k_shares(long long tiles, int kblocks_per_tile, int ctas, int tile, int max_shares,
                                      int* cta, int* slot, int* n_shares);

/* The 16 NF4 levels this library uses (host fp32[16]): the NormalFloat-4 code of the pages'
 * `quantization: 4bit` (guillermodelpino soup.yaml example), Dettmers et al. 2023. */
soup_status soup_nf4_codebook(float* out16);

/* ---- diagnostics ------------------------------------------------------------------------- */
/* The pages define none of these; they measure the library's own work.  The link the probe
 * times is the cost the pages name for streaming (guillermodelpino "Cuándo no te compensa":
 * moving layers costs speed). */
/* Host-to-device link probe: copies the model's page-locked layer-0 blob into a device layer
 * buffer `reps` times back to back on the streamer's copy stream (the exact path the streamer
 * uses) and returns the achieved GB/s (1e9 bytes/s) in *gbs.  Synchronises; the buffer used is
 * marked empty afterwards, so the next step reloads whatever it needs. */
soup_status soup_h2d_probe(soup_model* model, int reps, double* gbs);
soup_status soup_get_stats(soup_model* model, soup_stats* out);
soup_status soup_reset_stats(soup_model* model);
/* Live per-kernel profile.  While enabled, every launch a model call makes is bracketed by
 * CUDA events on the stream it runs on (the H2D layer copies on the streamer's copy stream)
 * and accumulated per category: launches, device milliseconds and the launch's algorithmic
 * work (flops of the dense contraction, bytes of its inputs and outputs).  Adds one event
 * pair per launch; soup_get_profile synchronises the recorded events.  Every step made while
 * enabled first times 8 empty launches the same way, reported as category "event_overhead":
 * the part of each launch's time that is the measurement's own. */
typedef struct soup_profile_entry {
  char name[32];
  long long launches;
  double total_ms;
  double flops;
  double bytes;
} soup_profile_entry;
soup_status soup_set_profiling(soup_model* model, int enabled);
/* Copies up to max_entries categories (those with launches) into out; *n_entries = count.
 * Clears the accumulated profile when reset != 0. */
soup_status soup_get_profile(soup_model* model, soup_profile_entry* out, int max_entries, int* n_entries, int reset);

/* Timed categories: brackets every launch of the named profile categories (names soup_get_profile
 * reports, comma-separated, e.g. "gemm_nf4_fwd,gemm_nf4_dx"; "all" for every category, layer
 * copies included) with a CUDA
 * event pair in ordinary model calls, including the CUDA graphs the layer calls replay (the
 * pair becomes two external event-record nodes of the graph, recorded on the stream the
 * kernel runs on at every replay).  Unlike soup_set_profiling it changes neither launch order
 * nor graph use nor stream concurrency, so it times launches as ordinary calls run them; the
 * event nodes themselves cost some microseconds per pair, measured by one empty launch at the
 * start of every layer call, bracketed the same way and reported by soup_get_timed_profile as
 * category "event_overhead" (not counted by soup_get_timed_category).  NULL or "" turns it off; an
 * unknown name is SOUP_ERR_INVALID_ARG.  Setting it clears the totals; graphs are captured
 * anew for the new setting (the first two calls of each layer after a change run eagerly /
 * capture, as at start-up). */
soup_status soup_set_timed_category(soup_model* model, const char* category);
/* Totals over the timed launches since the last reset, summed over the timed categories:
 * launches, device milliseconds (sum of the event pairs), algorithmic flops and bytes.  Waits
 * for the recorded events.  name holds the setting's first 31 characters ("" when none).
 * Clears the totals when reset != 0. */
soup_status soup_get_timed_category(soup_model* model, soup_profile_entry* out, int reset);
/* The same totals per category, in the layout of soup_get_profile (categories with launches,
 * up to max_entries; *n_entries = count).  Clears the totals when reset != 0. */
soup_status soup_get_timed_profile(soup_model* model, soup_profile_entry* out, int max_entries, int* n_entries,
                                   int reset);

/* Self-test of the failure path of every in-kernel wait.  Each wait of the library's kernels on
 * a shared-memory barrier is bounded (2 s): when the bound runs out the kernel sets the model's
 * device error word and runs to its end instead of hanging, and the next call that reads the
 * word returns SOUP_ERR_TIMEOUT.  This call launches one thread that waits, with the same wait
 * code, on a barrier that nothing ever arrives on, with a bound of limit_us microseconds (1 ..
 * 1000000); it returns after enqueueing on `stream`.  A soup_check_device (or the next
 * soup_step) then reports SOUP_ERR_TIMEOUT once, clears the word, and the model stays usable.
 * The pages have no counterpart: this is the library's own fault reporting. */
soup_status soup_selftest_bounded_wait(soup_model* model, int limit_us, void* stream);
/* Reads (and clears) the device error word; SOUP_ERR_TIMEOUT / SOUP_ERR_DEVICE_CHECK if set.
 * Synchronises `stream`.  The library's own fault reporting (no page counterpart). */
soup_status soup_check_device(soup_model* model, void* stream);
const char* soup_status_string(soup_status status);
const char* soup_last_error(const soup_model* model);

#ifdef __cplusplus
}
#endif

#endif /* SOUP_H_ */
