/*
 * bltdec.h -- C ABI of the Fast-BLT local-decoder engine (sm_100a).
 *
 * The engine runs the byte-level local decoder of Fast-BLT on one GPU:
 * BLT-D block diffusion with confidence unmasking, BLT-S autoregressive
 * drafts, BLT-DV diffusion drafts, and the greedy verification pass shared by
 * BLT-S and BLT-DV.  The global model, local encoder and entropy patcher are
 * NOT part of the engine: the caller supplies patch-boundary-derived latent
 * slots and the global latents O.
 *
 * Sources (page titles and sections):
 *   "Fast Byte Latent Transformer (Fast-BLT) 연구 소개" (discuss.pytorch.kr):
 *     - "계층적 BLT: 인코더, 글로벌 모델, 디코더": decoder layer equation
 *       B_l = D_{l-1} + W_o softmax(QK^T/sqrt(d_k)) V, D_l = DecoderTransformerLayer(B_l)
 *     - "BLT-D 추론": block decoding loop, prefix / latent caching
 *     - "BLT-D의 어텐션 마스크": latent rule and self-attention mask
 *     - "블록 언마스킹 전략": confidence-based unmasking with threshold alpha
 *     - "BLT-S와 BLT-DV": greedy verification (accept while x'_i == y_{i-1},
 *       replace the first mismatch, free byte when all match)
 *     - "BLT-S", "BLT-DV": the two drafting modes
 *
 * Conventions common to every call
 *   - Return value: BLT_OK (0) or a negative BLT_ERR_*.  Errors found on the
 *     host return at once and leave the handle unchanged; errors found on
 *     the device are written to the handle's status word and reported by
 *     blt_dec_sync().  blt_dec_last_error() gives a message.
 *   - Pointers marked "device" are CUDA device pointers owned by the caller;
 *     they are read or written by stream-ordered work on the handle's stream
 *     and must stay valid until that work completes.  Pointers marked "host"
 *     are read during the call only.
 *   - A handle is not thread-safe.  Calls are asynchronous with respect to
 *     the host unless stated otherwise.
 *   - Rows: a "row" is one byte position of one sequence run through the
 *     decoder.  A row's "latent slot" is the 0-based index of the one global
 *     latent its cross-attention sees: with patches numbered from 1, a byte
 *     of patch p sees o_{p-1}, except the last byte of a patch, which sees
 *     o_p; o_j is stored in slot j-1.  Slots must be < the sequence's latent
 *     count at the time the row is run.
 *   - Byte positions are 0-based and never reused; every sequence's decoded
 *     bytes sit at consecutive positions after its prefix.
 */
#ifndef BLTDEC_H
#define BLTDEC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BLT_OK 0
#define BLT_ERR_INVALID_ARG (-1) /* bad size, pointer, or argument combination */
#define BLT_ERR_NO_SPACE (-2)    /* KV page pool, latent capacity or row capacity exhausted */
#define BLT_ERR_STATE (-3)       /* call out of order (verify without a draft ...) */
#define BLT_ERR_CUDA (-4)        /* a CUDA runtime call failed */
#define BLT_ERR_STEP_LIMIT (-5)  /* masked positions left after max_steps passes (device) */
#define BLT_ERR_DEVICE (-6)      /* a device-side index check failed (device) */

#define BLT_W_F32 0  /* weights kept as two bf16 planes (hi + lo); fp32 KV cache */
#define BLT_W_BF16 1 /* weights kept as one bf16 plane (values rounded to bf16); bf16 KV cache */

#define BLT_DRAFT_AR 0        /* BLT-S: k autoregressive passes */
#define BLT_DRAFT_DIFFUSION 1 /* BLT-DV: confidence unmasking of a k-byte block */

/* Per-layer weight tensors, fp32, row-major PyTorch Linear layout [out, in]. */
#define BLT_LAYER_WQ_C 0      /* [d, d]   cross-attn query  (accepted, never read: one key per row) */
#define BLT_LAYER_WK_C 1      /* [d, dg]  cross-attn key    (accepted, never read: one key per row) */
#define BLT_LAYER_WV_C 2      /* [d, dg]  cross-attn value */
#define BLT_LAYER_WO_C 3      /* [d, d]   cross-attn output */
#define BLT_LAYER_NORM_C 4    /* [d]      cross-attn query RMSNorm gain (never read) */
#define BLT_LAYER_ATTN_NORM 5 /* [d]      pre-self-attention RMSNorm gain */
#define BLT_LAYER_WQKV 6      /* [3d, d]  rows q, k, v; head h owns rows h*dh..h*dh+dh-1 of each */
#define BLT_LAYER_WO 7        /* [d, d]   self-attention output */
#define BLT_LAYER_FFN_NORM 8  /* [d]      pre-FFN RMSNorm gain */
#define BLT_LAYER_W1 9        /* [F, d]   SwiGLU gate */
#define BLT_LAYER_W3 10       /* [F, d]   SwiGLU up */
#define BLT_LAYER_W2 11       /* [d, F]   SwiGLU down */
#define BLT_LAYER_NT 12

typedef struct blt_dec blt_dec_t; /* opaque; owns weights, KV pool, latent cache, scratch */

typedef struct {
  int32_t n_layers, d_model, n_heads, d_ffn, d_global;
  int32_t vocab;        /* 257: bytes 0..255 and the [MASK] id 256 */
  int32_t weight_dtype; /* BLT_W_F32 | BLT_W_BF16 */
  float rope_theta;     /* rotary base (rotate-half pairing) */
  float norm_eps;       /* RMSNorm epsilon */
  int32_t max_batch;    /* sequences in the handle */
  int32_t max_ctx;      /* byte positions per sequence, including drafts/blocks in flight */
  int32_t max_latents;  /* latent slots per sequence, including provisional ones */
  int32_t max_rows;     /* rows in one decoder pass (prefill is chunked to this) */
  int32_t max_block;    /* largest k / block size */
  int32_t page_tokens;  /* KV positions per page; multiple of 16 */
  int32_t kv_pages;     /* pages in the pool; 0 = enough for max_batch * max_ctx */
  int32_t attn_chunk;   /* keys per split-KV chunk; 0 = 128 */
  int32_t flags;        /* BLT_FLAG_* */
} blt_dec_config;

#define BLT_FLAG_TIME_PASSES 1 /* bracket the decoder passes of every call with CUDA events (counters.pass_ns) */
#define BLT_FLAG_PERSISTENT 2  /* run small passes (<= 16 rows) in the persistent pass kernel (one launch per call) */
#define BLT_FLAG_TEST_STALL 4  /* test only: in the persistent kernel, one output of the first pass's first O
                                  projection is never published and the waits give up after about a
                                  millisecond: the call's passes stop and blt_dec_sync reports
                                  BLT_ERR_DEVICE (exercises the bounded waits; never set in production) */
#define BLT_FLAG_TENSOR_CORES 8 /* passes of >= 128 rows (prefill chunks included) run their projections
                                   (QKV, O, SwiGLU, W2, head) on the tcgen05 GEMM (bf16 weights only).
                                   Results then agree with the GEMV path to rounding, not bit for bit.
                                   Costs a second, row-major bf16 copy of those weights. */

typedef struct {
  const float *embed;      /* host [vocab, d] */
  const float *head;       /* host [vocab, d]; row vocab-1 ([MASK]) is never predicted */
  const float *final_norm; /* host [d] */
  const float *const *layer; /* host: n_layers * BLT_LAYER_NT host pointers, index l*BLT_LAYER_NT + t */
} blt_dec_weights;

/* Rows the caller has committed but the engine has not cached, plus latents
 * that became available with them.  Sequence s owns rows
 * row_offsets[s] .. row_offsets[s+1]-1 (its next uncached positions, in
 * order) and latents latent_offsets[s] .. latent_offsets[s+1]-1 (appended to
 * its latent slots, in order). */
typedef struct {
  const uint8_t *bytes;          /* device [n_rows]            byte values */
  const int32_t *row_latent;     /* device [n_rows]            latent slot of each row */
  const int32_t *row_offsets;    /* host   [batch+1]           row_offsets[0] == 0 */
  const float *new_latents;      /* device [n_latents, d_global] fp32 (may be NULL when none) */
  const int32_t *latent_offsets; /* host   [batch+1]           latent_offsets[0] == 0 */
} blt_rows_in;

typedef struct {
  uint64_t passes;         /* decoder passes run (decoder NFE, batch-level) */
  uint64_t rows;           /* rows run through the decoder */
  uint64_t prefill_rows;   /* rows cached by blt_dec_prefill */
  uint64_t latents;        /* latents projected (global-model outputs consumed) */
  uint64_t calls;          /* C-ABI calls that ran decoder work */
  uint64_t weight_bytes;   /* weight bytes streamed by decoder passes (algorithmic) */
  uint64_t kv_read_bytes;  /* K/V bytes read by the self-attention of decoder passes (algorithmic; prefill excluded) */
  uint64_t kernel_launches; /* engine kernels launched (host count) */
  uint64_t timed_passes;   /* decoder passes inside timed calls (BLT_FLAG_TIME_PASSES) */
  uint64_t pass_ns;        /* summed device time of those calls' passes, ns (latent projection excluded) */
  uint64_t persistent_calls; /* calls whose decoder passes ran in the persistent kernel (BLT_FLAG_PERSISTENT) */
  uint64_t prefill_kv_read_bytes; /* K/V bytes read by the self-attention of prefill chunks (algorithmic) */
  uint64_t tc_gemms;       /* projections run on the tcgen05 GEMM (BLT_FLAG_TENSOR_CORES) */
} blt_dec_counters;

/* Create an engine.  Copies and re-lays out the weights on the device
 * (bf16 tiles in tensor-core fragment order), allocates the paged KV pool,
 * the latent cache and all scratch.  cuda_stream: a cudaStream_t (NULL = a
 * new non-blocking stream owned by the engine).  Synchronous.
 * Errors: INVALID_ARG (shape not supported: d_model, d_global, d_ffn multiples
 * of 128; d_model/n_heads a multiple of 16 and <= 128; vocab 257), CUDA. */
int blt_dec_init(const blt_dec_config *cfg, const blt_dec_weights *w, void *cuda_stream, blt_dec_t **out);

/* Cache the K/V of committed rows with causal attention (section "BLT-D 추론":
 * the clean prefix is cached).  Rows are run in chunks of max_rows.  The
 * latents are committed before any row runs.  out_logits (device, may be
 * NULL): [n_rows, 256] next-byte logits of every row.
 * Errors: INVALID_ARG, NO_SPACE, STATE (a draft is waiting for verification). */
int blt_dec_prefill(blt_dec_t *h, int batch, const blt_rows_in *rows, float *out_logits);

/* blt_dec_prefill, with no allocation of its own.  (The paper has no
 * counterpart: this is an engineering entry point.)
 *
 * Same inputs, outputs, semantics and errors as blt_dec_prefill, but the
 * per-call scratch of the decoder passes (activations, split-KV attention
 * partials, logits, the row plan, the latent-projection temporary) lives in
 * one file-scope static device arena instead of the handle's scratch, and
 * the call makes no cudaMalloc, cudaFree or other allocating call.  Callers
 * that cannot allocate device memory at call time use it: a serving process
 * that sized the handle small (max_rows, the scratch blt_dec_init allocates)
 * and runs under a device-memory budget that is already spent, or a host
 * thread that must not allocate once set-up is over, can still prefill in
 * 32-row chunks.
 *
 * Limits (else INVALID_ARG): d_model <= 1024, d_ffn <= 4096, n_heads <= 16,
 * head dim <= 64, n_layers * d_model <= 32768 (the latent-projection
 * temporary), attn_chunk 128 (the default), and each sequence's cached
 * length plus its rows <= 4096 positions.  Its 32-row chunks always take the
 * GEMV kernels, so the logits and the KV cache it writes are bit-identical to
 * blt_dec_prefill's on a handle without BLT_FLAG_TENSOR_CORES (a row's
 * arithmetic does not depend on which rows share its pass); with that flag,
 * blt_dec_prefill's chunks of >= 128 rows take the tcgen05 GEMM and agree to
 * rounding.  The arena is about 5.2 MB and every
 * GPU that loads the library holds it until the process exits.
 * The first call on a device resolves the arena's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Every call shares the one arena, which keeps
 * the last call's contents (nothing in it needs to start at zero): calls that
 * overlap on the GPU -- on different streams or handles -- race. */
int blt_dec_prefill_noalloc(blt_dec_t *h, int batch, const blt_rows_in *rows, float *out_logits);

/* BLT-D: fill one masked block of k bytes per sequence ("BLT-D 추론",
 * "블록 언마스킹 전략").  The pending rows ride, causally, in the first pass
 * and are cached.  Block rows sit at the next k positions, attend the whole
 * clean prefix and each other (bidirectional), and see the newest committed
 * latent; each pass commits every masked position whose confidence (largest
 * softmax probability over the 256 bytes) is >= alpha, or the single most
 * confident masked position when none is (ties: lowest position; argmax
 * ties: lowest byte).  Passes repeat on the device until every block is full
 * (at most max_steps; 0 means k).  Block bytes are NOT cached: the caller
 * commits them and passes them back as pending rows of the next call.
 * out_block  device [batch, k] u8        the filled blocks
 * out_steps  device [batch] i32 (NULL ok) passes each sequence needed
 * out_logits device (NULL ok) [max_steps, batch, k, 256] logits of the block
 *            rows in every pass (entries of finished sequences untouched)
 * A draft waiting for verification is discarded (its provisional K/V are
 * overwritten; the pending rows of its call stay cached).
 * Device error: STEP_LIMIT.  Host errors: INVALID_ARG, NO_SPACE. */
int blt_dec_diffuse_block(blt_dec_t *h, int batch, const blt_rows_in *pending, int k, float alpha, int max_steps,
                          uint8_t *out_block, int32_t *out_steps, float *out_logits);

/* BLT-D with entropy-bounded (EB) sampling instead of the confidence rule
 * ("블록 언마스킹 전략", EB sampling; the wangzhan123.com page, section on the
 * two unmasking rules).  Everything is as in blt_dec_diffuse_block except the
 * per-pass choice: the still-masked positions are ordered by the entropy
 * (nats) of their predicted distribution over the 256 bytes, lowest first
 * (equal entropies: lower position first); running sums of those entropies
 * are taken in that order (fp32) and every position whose running sum is
 * <= gamma is committed, and always at least the first.  Committed bytes are
 * the greedy argmax.  gamma: finite, >= 0 (else INVALID_ARG).  Same outputs,
 * ownership and errors as blt_dec_diffuse_block. */
int blt_dec_diffuse_block_eb(blt_dec_t *h, int batch, const blt_rows_in *pending, int k, float gamma, int max_steps,
                             uint8_t *out_block, int32_t *out_steps, float *out_logits);

/* Draft k bytes per sequence after the committed ones ("BLT-S", "BLT-DV").
 * Every sequence needs at least one pending row: the last pending row's
 * greedy prediction is y_l of the verification.
 * BLT_DRAFT_AR: k passes; pass 1 runs the pending rows, pass t > 1 runs the
 * draft byte t-1 at the next position, seeing the newest committed latent.
 * BLT_DRAFT_DIFFUSION: a k-byte masked block filled as in
 * blt_dec_diffuse_block with threshold alpha (alpha 0: one pass).
 * Draft K/V are provisional (overwritten by verification).  A draft already
 * waiting is discarded, so a k = 1 AR draft whose byte the caller commits
 * without verification (it is y_l itself) is one plain greedy AR step.
 * out_draft  device [batch, k] u8
 * out_logits device (NULL ok): AR [k, batch, 256]; DIFFUSION as diffuse_block.
 * Errors: INVALID_ARG, NO_SPACE. */
int blt_dec_draft(blt_dec_t *h, int batch, const blt_rows_in *pending, int mode, int k, float alpha, int max_steps,
                  uint8_t *out_draft, float *out_logits);

/* Greedy verification of the waiting draft ("BLT-S와 BLT-DV").  One causal
 * pass runs the k draft bytes at their positions with the re-patched latent
 * slots (draft_row_latent); new_latents/latent_offsets add the latents of
 * patches the draft closes (provisional).  With y_l the prediction of the last
 * committed row and y_{l+t} that of draft row t, the accepted length a is the
 * number of leading draft bytes with draft[i] == y_{l+i}; the next byte is
 * y_{l+a} (a correction, or the free byte when a == k).  The a accepted rows'
 * K/V become cached; latents of patches closed by accepted bytes are kept.
 * The caller commits draft[0..a) and the next byte; the next byte is the
 * pending row of the following call.
 * draft_row_latent device [batch, k] i32; new_latents device (NULL ok);
 * latent_offsets host [batch+1] (NULL = none)
 * out_accepted device [batch] i32; out_next device [batch] u8;
 * out_logits device (NULL ok) [batch, k, 256].
 * Errors: INVALID_ARG, NO_SPACE, STATE (no draft waiting). */
int blt_dec_verify_accept(blt_dec_t *h, const int32_t *draft_row_latent, const float *new_latents,
                          const int32_t *latent_offsets, int32_t *out_accepted, uint8_t *out_next, float *out_logits);

/* ---- stochastic decoding -------------------------------------------------
 * Fast-BLT (discuss.pytorch.kr), "블록 언마스킹 전략": the unmasking rules can be
 * combined with top-p sampling; "BLT-S와 BLT-DV": with a non-zero temperature the
 * verification extends through rejection sampling (the page evaluates greedy
 * decoding only).  Definitions used here (the page gives none):
 *   dist(z) = softmax(z / temperature) over the 256 byte logits, bytes ranked by
 *     probability (ties: lower byte first), the shortest leading run whose
 *     cumulative probability reaches top_p kept and renormalised;
 *   a draw with uniform u = the smallest byte b whose cumulative probability
 *     (bytes in increasing order) exceeds u.
 * Random numbers are inputs: `uniforms` is a device array [batch][2 k + 1] of
 * values in [0, 1) (k: the call's block / draft size; for verification the
 * waiting draft's), owned by the caller and read during the call's stream work.
 * These calls run on the per-phase kernels (never the persistent one). */
typedef struct {
  float temperature;     /* > 0 */
  float top_p;           /* in (0, 1] */
  const float *uniforms; /* device [batch][2 k + 1] */
} blt_sampling;

#define BLT_UNMASK_CONFIDENCE 0 /* threshold = alpha */
#define BLT_UNMASK_EB 1         /* threshold = gamma (entropy bound, nats) */

/* blt_dec_diffuse_block (unmask = CONFIDENCE) or blt_dec_diffuse_block_eb
 * (unmask = EB), with the positions each pass commits chosen by that rule and
 * their bytes drawn from dist(logits of their rows) with uniforms[s][i] for
 * block position i.  Errors: those of the greedy call, INVALID_ARG for bad
 * sampling parameters. */
int blt_dec_diffuse_block_sampled(blt_dec_t *h, int batch, const blt_rows_in *pending, int k, float threshold, int unmask,
                                  int max_steps, const blt_sampling *sampling, uint8_t *out_block, int32_t *out_steps,
                                  float *out_logits);

/* blt_dec_draft with drawn bytes: BLT_DRAFT_AR draws draft byte t from
 * dist(logits of pass t's row) with uniforms[s][t]; BLT_DRAFT_DIFFUSION draws
 * the bytes the unmasking commits, as blt_dec_diffuse_block_sampled (confidence
 * rule).  The distribution each draft byte was drawn from, and the target of
 * draft slot 0 (dist of the last committed byte's row), are kept for
 * blt_dec_verify_sampled. */
int blt_dec_draft_sampled(blt_dec_t *h, int batch, const blt_rows_in *pending, int mode, int k, float alpha, int max_steps,
                          const blt_sampling *sampling, uint8_t *out_draft, float *out_logits);

/* Verification of a blt_dec_draft_sampled draft by rejection sampling.  The
 * causal pass is blt_dec_verify_accept's; then per sequence, for slots
 * t = 0..k-1 with draft byte x_t, draft distribution q_t and target p_t (slot 0:
 * the kept target; slot t > 0: dist of verification row t - 1): x_t is
 * accepted while uniforms[s][t] < min(1, p_t(x_t) / q_t(x_t)); at the first
 * rejection out_next[s] is drawn from max(p_t - q_t, 0) renormalised (p_t if
 * that is zero) with uniforms[s][k + t]; if all k are accepted, out_next[s] is
 * drawn from dist(row k - 1) with uniforms[s][2 k].  out_accepted / out_next /
 * KV commit as in blt_dec_verify_accept.  Errors: as blt_dec_verify_accept;
 * STATE when the waiting draft was not drawn. */
int blt_dec_verify_sampled(blt_dec_t *h, const int32_t *draft_row_latent, const float *new_latents,
                           const int32_t *latent_offsets, const blt_sampling *sampling, int32_t *out_accepted,
                           uint8_t *out_next, float *out_logits);

/* Set sequences' cached length and committed latent count (host arrays
 * [batch]; -1 keeps a value).  Values may only shrink.  Drops a waiting draft.
 * Synchronous with respect to the handle's stream.  Errors: INVALID_ARG. */
int blt_dec_rewind(blt_dec_t *h, int batch, const int32_t *kv_len, const int32_t *n_latents);

/* Read the counters (waits for the handle's stream). */
int blt_dec_stats(blt_dec_t *h, blt_dec_counters *out);

/* Host <-> device copies on the handle's stream, for the rows, latents and
 * outputs of the calls above (plain runtime helpers; no decoder work).
 * blt_dec_upload: copies n bytes from host memory src (any memory; it is
 * read before the call returns, so the caller may reuse it at once) to device
 * memory dst, through one of the handle's pinned bounce buffers; the device
 * copy is queued on the stream (later calls on the handle see it).
 * blt_dec_download: copies n bytes from device memory src to host memory dst
 * after all queued work; returns once dst holds them.  Both: n = 0 does no
 * copy; the device pointers must be valid for n bytes.  Errors: INVALID_ARG
 * (NULL pointer with n > 0), CUDA. */
int blt_dec_upload(blt_dec_t *h, void *dst_device, const void *src_host, size_t n);
int blt_dec_download(blt_dec_t *h, void *dst_host, const void *src_device, size_t n);

/* Wait for all queued work; returns BLT_OK or the device status word
 * (BLT_ERR_STEP_LIMIT, BLT_ERR_DEVICE) and clears it. */
int blt_dec_sync(blt_dec_t *h);

/* Message of the last error on this handle ("" if none).  Valid until the next call. */
const char *blt_dec_last_error(blt_dec_t *h);

/* Free everything the handle owns (waits for its stream first). */
void blt_dec_free(blt_dec_t *h);

#ifdef __cplusplus
}
#endif
#endif /* BLTDEC_H */
