/*
 * fs.h — C ABI of libfs: the forward pass of a dense Qwen3-class decoder-only
 * transformer on one NVIDIA B200 (sm_100a), run as prefill and as KV-cached
 * autoregressive decode.
 *
 * The pass ("Milestones", M2 Forward pass -> logits; "Coming back to Failed
 * Star", data-flow figure under "Second sitting"):
 *   ids -> embedding [S,H] -> L blocks of
 *     RMSNorm -> Q/K/V projection -> per-head q/k RMSNorm -> RoPE ->
 *     causal GQA attention over the KV cache -> O projection -> residual ->
 *     RMSNorm -> SwiGLU MLP -> residual
 *   -> final RMSNorm of the last row -> tied LM head -> logits[V]
 *   -> greedy selection (argmax, lowest id on exact ties).
 *
 * Conventions for every call:
 *  - Every call returns an fs_status: FS_OK (0) or a negative error code. No
 *    call throws, aborts or prints. fs_last_error_string() describes the last
 *    error raised on the calling thread.
 *  - "device pointer" means memory the CUDA device can read (cudaMalloc,
 *    torch CUDA tensors). Device pointers handed to the library must be
 *    16-byte aligned (FS_ERR_ALIGN otherwise), except int32 token and argmax
 *    arrays, which need 4-byte alignment.
 *  - Token arrays may be host or device memory; the library asks the CUDA
 *    runtime which it is. Host token arrays are validated on the host
 *    (FS_ERR_TOKEN before anything runs); device token arrays are validated on
 *    the device: an id outside [0, V) is replaced by 0 and the model's device
 *    error word is set, reported by fs_device_error().
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream). Calls that take a stream only enqueue work on it and return
 *    without waiting, except fs_greedy, which waits for its result.
 *  - Weights are caller-owned device memory that must outlive the model.
 *    Memory the library allocates (RoPE table, workspace, KV pages, fp16
 *    shadow weights for prefill) is library-owned and freed by the matching
 *    destroy/free call.
 *  - A model or KV handle must not be used from two host threads at once.
 */
#ifndef FS_H
#define FS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t fs_status;

#define FS_OK 0
#define FS_ERR_INVALID (-1)     /* bad config, size or argument value */
#define FS_ERR_NULL (-2)        /* a required pointer is NULL */
#define FS_ERR_ALIGN (-3)       /* a device pointer is not 16-byte aligned */
#define FS_ERR_OOM (-4)         /* a device allocation failed */
#define FS_ERR_EMPTY (-5)       /* zero tokens where at least one is required */
#define FS_ERR_TOKEN (-6)       /* a host token id is outside [0, vocab) */
#define FS_ERR_CONTEXT (-7)     /* the call would exceed max_pos or KV capacity */
#define FS_ERR_CUDA (-8)        /* a CUDA runtime call or a launch failed */
#define FS_ERR_SEQ (-9)         /* sequence index out of range or repeated in a batch */
#define FS_ERR_DEVICE (-10)     /* a kernel set the device error word */
#define FS_ERR_UNSUPPORTED (-11) /* a shape outside what the kernels cover */

/* Weight formats of the linear layers (the embedding / LM head is always bf16). */
#define FS_WEIGHT_BF16 0
/* Q8_0 ("ferrite", "What it does": one of the dequantised formats): blocks of
 * 32 consecutive weights along the input axis, w = q * s with q int8 in
 * [-127, 127] and one fp16 scale s per block. Stored struct-of-arrays:
 * codes int8 [N, K] row-major, scales fp16 [N, K/32] row-major. */
#define FS_WEIGHT_Q8_0 1

/* Why fs_greedy stopped ("Coming back to Failed Star", "Next: one complete
 * deterministic generation arc", Stopping / Budget). */
#define FS_STOP_EOS 1     /* the selected id is an EOS id; it is included in the output */
#define FS_STOP_BUDGET 2  /* max_new ids were produced (also when max_new == 0) */
#define FS_STOP_CONTEXT 3 /* the next forward would exceed max_pos or the KV capacity;
                             the last allowed forward's prediction is included */

/* Model shape ("Coming back to Failed Star", shape legend: L=28, H=1024,
 * 16 query heads, 8 KV heads, d=128, I=3072, V=151936 for Qwen3-0.6B).
 * Requirements: n_q_heads % n_kv_heads == 0; head_dim even and <= 128;
 * hidden, ffn and n_q_heads*head_dim multiples of 64 (multiples of 32 are
 * also what Q8_0 needs); 1 <= max_pos <= 1<<20. */
typedef struct fs_config {
  int32_t n_layers;   /* L */
  int32_t hidden;     /* H */
  int32_t n_q_heads;  /* query heads */
  int32_t n_kv_heads; /* key/value heads (GQA groups) */
  int32_t head_dim;   /* d */
  int32_t ffn;        /* I, SwiGLU inner width */
  int32_t vocab;      /* V */
  float rms_eps;      /* RMSNorm epsilon (1e-6 for the Qwen3 family) */
  double rope_theta;  /* RoPE base (1e6 for the Qwen3 family) */
  int32_t max_pos;    /* positions 0 .. max_pos-1 may be used */
  int32_t weight_format; /* FS_WEIGHT_BF16 or FS_WEIGHT_Q8_0 for the 7 linear layers */
} fs_config;

/* One linear layer, row-major [out, in] (a Linear stored [out,in] maps
 * [S,in] to [S,out]: "Coming back to Failed Star", "Second sitting").
 * bf16: `data` = bf16 [out, in], `scales` = NULL.
 * Q8_0: `data` = int8 codes [out, in], `scales` = fp16 [out, in/32]. */
typedef struct fs_linear {
  const void* data;
  const void* scales;
} fs_linear;

/* Device pointers of one block. Norm gains are bf16: attn_norm and ffn_norm
 * [H], q_norm and k_norm [head_dim]. wq [nq*d, H], wk and wv [nkv*d, H],
 * wo [H, nq*d], wg and wu [I, H], wd [H, I]. No biases. */
typedef struct fs_layer_weights {
  fs_linear wq, wk, wv, wo, wg, wu, wd;
  const void* attn_norm;
  const void* ffn_norm;
  const void* q_norm;
  const void* k_norm;
} fs_layer_weights;

typedef struct fs_weights {
  const void* embed;       /* bf16 [V, H]; also the tied LM head */
  const void* final_norm;  /* bf16 [H] */
  const fs_layer_weights* layers; /* HOST array of n_layers entries */
} fs_weights;

typedef struct fs_model fs_model;
typedef struct fs_kv fs_kv;

/* Create a model on the current CUDA device from a config and caller-owned
 * device weights. Validates the config, every pointer (non-NULL, 16-byte
 * aligned device memory) and builds the RoPE cos/sin table on the host in fp64
 * (rounded to fp32). Allocates the library-owned workspace. When the
 * persistent decode kernel covers the shape, it also makes library-owned
 * transposed copies of every block's wo and wd ([in, out]; Q8_0: codes and
 * scales), read by the decode kernel in place of the caller's: the weights
 * must not change after this call.
 * Errors: FS_ERR_NULL, FS_ERR_INVALID, FS_ERR_ALIGN, FS_ERR_UNSUPPORTED,
 * FS_ERR_OOM, FS_ERR_CUDA. On error *out is set to NULL. */
fs_status fs_model_create(const fs_config* cfg, const fs_weights* weights, fs_model** out);

/* Free library-owned memory of a model (weights are the caller's). NULL is a no-op.
 * The caller must make sure no work using the model is still running.
 * No page defines teardown; this is the release half of the device buffers
 * the engine brings up ("Failed Star / fs — Milestones", M5: device, queue,
 * buffers and pipelines owned by the engine). */
void fs_model_destroy(fs_model* model);

/* Allocate a paged bf16 KV cache for up to `max_seqs` sequences of up to
 * `max_tokens_per_seq` positions each ("Milestones", M4 KV cache: K/V per
 * layer so decode does one token of work). Pages hold 64 positions; each
 * sequence owns ceil(max_tokens_per_seq/64) pages reached through a block
 * table. K is stored after q/k-norm and RoPE. Every sequence starts empty.
 * The pages are zeroed: slots past a sequence's length always hold finite
 * values (the attention kernels read whole pages and weight those slots by
 * exact zeros; values imported with fs_kv_import must be finite too).
 * Errors: FS_ERR_NULL, FS_ERR_INVALID, FS_ERR_OOM. */
fs_status fs_kv_alloc(const fs_model* model, int32_t max_seqs, int32_t max_tokens_per_seq,
                      fs_kv** out);

/* Free a KV cache. NULL is a no-op. No work using it may still be running.
 * ("Failed Star / fs — Milestones", M4: the cache is memory-only, so it lives
 * exactly as long as this object; nothing is persisted.) */
void fs_kv_free(fs_kv* kv);

/* Mark sequence `seq` empty (length 0). Waits for the device to go idle.
 * ("Failed Star / fs — Milestones", M4: a new generation on the sequence
 * starts from an empty cache; the pages are reused, not freed.) */
fs_status fs_kv_reset(fs_kv* kv, int32_t seq);

/* Current length (positions stored) of sequence `seq`, into *len (host). */
fs_status fs_kv_length(const fs_kv* kv, int32_t seq, int32_t* len);

/* Copy caller K/V into sequence `seq`, layer `layer`, positions
 * [pos0, pos0+n) ("Failed Star / fs — Milestones", M4: cached and uncached
 * outputs must agree, so a cache state has to be loadable and readable from
 * outside the forward; import also sets up a long pre-filled context without
 * running its prefill). `k` and `v` are device bf16 arrays in logical layout
 * [n, n_kv_heads, head_dim] holding stored values (already normalised and
 * rotated). The sequence length becomes max(length, pos0+n) once every layer
 * is imported — the caller states it with fs_kv_set_length.
 * Errors: FS_ERR_NULL, FS_ERR_SEQ, FS_ERR_CONTEXT (beyond capacity), FS_ERR_CUDA. */
fs_status fs_kv_import(fs_kv* kv, int32_t seq, int32_t layer, int32_t pos0, int32_t n,
                       const void* k, const void* v, void* stream);

/* The reverse of fs_kv_import: device bf16 [n, n_kv_heads, head_dim] out
 * (the same M4 passage: the stored K/V are compared with an uncached
 * recompute). Errors: as fs_kv_import. */
fs_status fs_kv_export(const fs_kv* kv, int32_t seq, int32_t layer, int32_t pos0, int32_t n,
                       void* k, void* v, void* stream);

/* Set the length of sequence `seq` (after fs_kv_import). 0 <= len <= capacity. */
fs_status fs_kv_set_length(fs_kv* kv, int32_t seq, int32_t len);

/* Prefill: run `n_tokens` ids of sequence `seq` at positions
 * length .. length+n_tokens-1, append their K/V, and write the logits of the
 * LAST row ("Coming back to Failed Star": only the final row is projected to
 * [V]) as fp32 [V] into `logits_out` (device, may be NULL) and its greedy
 * choice into `argmax_out` (device int32 [1], may be NULL).
 * Errors: FS_ERR_EMPTY (n_tokens == 0), FS_ERR_TOKEN (host ids only),
 * FS_ERR_CONTEXT, FS_ERR_SEQ, FS_ERR_NULL, FS_ERR_CUDA. */
fs_status fs_prefill(fs_model* model, fs_kv* kv, int32_t seq, const int32_t* tokens,
                     int32_t n_tokens, float* logits_out, int32_t* argmax_out, void* stream);

/* Decode one token for each of `batch` distinct sequences (ferrite, status
 * section: forward() run at consecutive positions on the same cache, each
 * output depending on the context stored so far; "Failed Star / fs —
 * Milestones", M4: decode does one token of work): sequence seqs[b]
 * (HOST array) takes token tokens[b] at its current length, appends its K/V
 * and gets logits fp32 [batch, V] (device, row b for seqs[b]; may be NULL) and
 * its greedy choice argmax_out[b] (device int32 [batch]; may be NULL).
 * `tokens` may be the previous step's argmax_out, which keeps a greedy loop
 * on the device. 1 <= batch <= 64.
 * Errors: FS_ERR_EMPTY, FS_ERR_SEQ, FS_ERR_TOKEN, FS_ERR_CONTEXT, FS_ERR_NULL,
 * FS_ERR_CUDA. */
fs_status fs_decode_step(fs_model* model, fs_kv* kv, const int32_t* seqs, const int32_t* tokens,
                         int32_t batch, float* logits_out, int32_t* argmax_out, void* stream);

/* One forward over a mixed batch of prefill chunks and decode rows
 * ("Failed Star / fs — Milestones", M4 KV cache: cached K/V per layer, so a
 * sequence's new tokens cost one token of work each, whichever call they
 * arrive in). Segment i appends n_tokens[i] >= 1 ids of sequence seqs[i] at
 * its current length (a prefill chunk when n_tokens[i] > 1, a decode row when
 * 1); `seqs` and `n_tokens` are HOST arrays of n_seqs distinct sequences;
 * `tokens` (host or device int32) holds the segments' ids back to back. Each
 * row attends to its own sequence's cache and the rows before it in its
 * segment. Writes the logits of each segment's LAST row to `logits_out`
 * (device fp32 [n_seqs, vocab], row i for segment i; may be NULL) and their
 * greedy ids to `argmax_out` (device int32 [n_seqs]; may be NULL). Runs the
 * general (any rows) kernels. A debug capture armed for this call holds the
 * rows in processing order: every segment's rows but the last, segment by
 * segment, then the segments' last rows. 1 <= sum of n_tokens <= 64.
 * Errors: FS_ERR_NULL, FS_ERR_EMPTY, FS_ERR_SEQ, FS_ERR_CONTEXT,
 * FS_ERR_INVALID, FS_ERR_TOKEN, FS_ERR_ALIGN, FS_ERR_CUDA. */
fs_status fs_forward_batch(fs_model* model, fs_kv* kv, const int32_t* seqs,
                           const int32_t* n_tokens, int32_t n_seqs, const int32_t* tokens,
                           float* logits_out, int32_t* argmax_out, void* stream);

/* Greedy continuation of `prompt` (n_prompt ids, host or device) on sequence
 * `seq`, following "Coming back to Failed Star", "Next: one complete
 * deterministic generation arc": no implicit BOS; n_prompt == 0 is
 * FS_ERR_EMPTY; max_new == 0 runs nothing and stops with FS_STOP_BUDGET; each
 * step selects the argmax (lowest id on exact ties); stops on an id in
 * eos_ids (HOST array, n_eos may be 0 = never), on max_new ids, or when the
 * next forward would pass max_pos or the KV capacity. Writes the generated ids
 * to out_tokens (host or device int32 [max_new]), their count to *n_out and
 * the reason to *stop_reason (both host). The sequence must be empty or hold
 * earlier context; the prompt is appended to it. Waits for completion.
 * Errors: as fs_prefill / fs_decode_step, FS_ERR_DEVICE. */
fs_status fs_greedy(fs_model* model, fs_kv* kv, int32_t seq, const int32_t* prompt,
                    int32_t n_prompt, int32_t max_new, const int32_t* eos_ids, int32_t n_eos,
                    int32_t* out_tokens, int32_t* n_out, int32_t* stop_reason, void* stream);

/* Seeded sampling of one id per row ("Coming back to Failed Star", "Next:
 * one complete deterministic generation arc": after greedy, temperature, then
 * top-k, then top-p, as explicit filters; "Failed Star / fs — Milestones",
 * M3). For each of `rows` rows of `logits` (device fp32 [rows, vocab]):
 * divide by `temperature`; rank ids by logit descending, ties to the lowest
 * id; keep the first `top_k` (0 or >= the finite count keeps all); over those,
 * keep the shortest prefix of the ranking whose softmax mass reaches `top_p`
 * (1 keeps all); renormalise; draw u in [0, 1) and return the first kept id
 * in ascending id order whose cumulative probability exceeds u. u is the top
 * 24 bits of the first word of Philox4x32-10 (Salmon et al., SC'11) with key
 * = `seed` (low word first) and counter = (step low word, row, step high
 * word, 0), times 2^-24. Non-finite logits are never drawn; a row with none
 * finite gives id 0. `temperature` == 0 is greedy selection (argmax, lowest
 * id on ties; top_k / top_p ignored). Probabilities are summed as exact
 * fixed-point integers (units of 2^-32 of the largest), so the result does
 * not depend on the order of summation. out_ids: device int32 [rows].
 * Requirements: 1 <= rows <= 64, temperature finite and >= 0, top_k >= 0,
 * 0 < top_p <= 1. Errors: FS_ERR_NULL, FS_ERR_INVALID, FS_ERR_ALIGN,
 * FS_ERR_CUDA. */
fs_status fs_sample(fs_model* model, const float* logits, int32_t rows, float temperature,
                    int32_t top_k, float top_p, uint64_t seed, uint64_t step, int32_t* out_ids,
                    void* stream);

/* fs_greedy with the next id drawn by fs_sample from each forward's last-row
 * logits instead of the argmax: generated id i (0-based) uses counter step i,
 * row 0. `temperature` == 0 is exactly fs_greedy. Same stop rules, outputs
 * and errors as fs_greedy, plus the argument checks of fs_sample. */
fs_status fs_generate(fs_model* model, fs_kv* kv, int32_t seq, const int32_t* prompt,
                      int32_t n_prompt, int32_t max_new, const int32_t* eos_ids, int32_t n_eos,
                      float temperature, int32_t top_k, float top_p, uint64_t seed,
                      int32_t* out_tokens, int32_t* n_out, int32_t* stop_reason, void* stream);

/* Debug: the next fs_prefill or fs_decode_step also writes the residual
 * stream before block 0 and after every block into `hidden` (device fp32
 * [(L+1), max_rows, H]): slot l, row r holds row r of the call (token r of a
 * prefill, batch row r of a decode) after l blocks; rows beyond max_rows are
 * not captured. One-shot: capture is disarmed after that call. NULL disarms. */
fs_status fs_debug_capture(fs_model* model, float* hidden, int32_t max_rows);

/* Debug: run block `layer` alone on `rows` rows of sequence `seq` at positions
 * length .. length+rows-1, from the residual-stream input h_in (device fp32
 * [rows, H]) to the block output h_out (device fp32 [rows, H]). It uses the
 * kernels the product path uses for that row count (one row: the persistent
 * decode kernel), reads the layer's cached K/V of earlier positions and writes
 * the layer's K/V for these positions; the sequence length is not changed.
 * Used to measure each block's own error given a reference input.
 * Errors: FS_ERR_NULL, FS_ERR_SEQ, FS_ERR_INVALID, FS_ERR_CONTEXT, FS_ERR_ALIGN. */
fs_status fs_debug_block(fs_model* model, fs_kv* kv, int32_t seq, int32_t layer,
                         const float* h_in, int32_t rows, float* h_out, void* stream);

/* Debug: the next decode step that runs on a persistent decode kernel
 * records timestamps into `buf` (device uint64 [SMs][n_layers+1][16]): per
 * CTA and block, the SM's cycle counter (clock64) at points of the step. Row
 * n_layers holds the tail and, in slots 12..15, the CTA's %globaltimer (ns)
 * and cycle counter at kernel start (12, 13) and end (14, 15), which place the
 * cycle stamps on a common time base. Slots per kernel (fs_debug_decode_kernel):
 * cooperative (1): 0 start of the QKV phase, 11 this CTA's slice of its input
 * reduced, 1 its input loaded, 2 QKV rows done, 3 start of the attention
 * phase, 4 q/k/v of the first batch row ready, 13 its keys done, 5 attention
 * merged, 6 O-projection share added, 7 start of the MLP phase, 12 this CTA's
 * slice of its input reduced, 8 its input loaded, 9 gate/up rows done, 10
 * down share added; tail 0 start, 11 slice of its input reduced, 1 input
 * loaded, 2 LM-head rows done, 3 the producer's last copy issued, 4 greedy
 * ids folded.
 * cluster (2): 0 block begins, 1 block input exchanged, 2 QKV rows done, 3
 * q/k/v exchanged, normed and rotated, 4 keys done and states sent, 5
 * attention merged and exchanged, 6 O shares published, 7 MLP input
 * exchanged, 8 gate/up and SwiGLU done, 9 activations exchanged, 10 down
 * shares published; tail 0 start, 1 input exchanged, 2 LM-head rows done, 3
 * the producer's last copy issued, 4 greedy ids folded.
 * row-split (3): 0 start of the QKV phase, 1 its input loaded, 8 QKV rows
 * done, 12 an attention item begins, 2 its q/k/v loaded, 13 q/k normed and
 * rotated, K/V appended, 14 its keys done, 15 the warps' states merged, 9
 * attention merged (across splits too), 3 start of the O phase, 4 its input
 * loaded, 10 start of the gate/up phase, 5 its input loaded, 11 start of the
 * down phase, 6 its input loaded, 7 block done; tail 0 start, 1 input
 * loaded, 2 the producer's first LM-head copy, 3 its last copy issued, 6
 * LM-head rows done, 7 greedy ids folded.
 * Slots a CTA never reaches are left as they were. One-shot; NULL disarms.
 * Timing only: no work changes. */
fs_status fs_debug_trace(fs_model* model, uint64_t* buf);

/* Debug: the time limit of every wait inside the persistent decode kernel
 * (a CTA waiting for another CTA's output or for a weight copy), `wait_ns`
 * in [1 us, 60 s], default 1 s, for all later steps. When a wait runs out
 * the kernel stops waiting everywhere, returns, and sets the device error
 * word to 3 (fs_device_error, which also clears the kernel's exchange state;
 * fs_greedy reports FS_ERR_DEVICE). `withhold_layer` >= 0 makes the next
 * step on that kernel never publish one of block `withhold_layer`'s hand-offs
 * between CTAs (the cooperative kernel: its Q/K/V projections; the cluster
 * kernel: its output-projection shares), so the waits for them run out (a
 * test of that path; the step's outputs are then undefined); -1 withholds
 * nothing. Errors: FS_ERR_NULL, FS_ERR_INVALID. */
fs_status fs_debug_wait_limit(fs_model* model, uint64_t wait_ns, int32_t withhold_layer);

/* Debug: which decode path later steps of 1..4 rows take. 0 (default): a
 * batch of 1 takes the row-split persistent kernel where its weight ring
 * holds a stage per consumer warp; other batches (and shapes it does not
 * cover) take the cluster kernel (clusters of 16 or 8 CTAs per kv head, on
 * shapes and devices it covers), else the cooperative persistent kernel, else
 * the general kernel sequence; 1: the cooperative kernel, else general; 2:
 * the general sequence only; 3: the row-split kernel, else general; 4: the
 * cluster kernel, else general. For comparing the paths in tests and
 * benchmarks; every path computes the same forward.
 * Errors: FS_ERR_NULL, FS_ERR_INVALID. */
fs_status fs_debug_decode_path(fs_model* model, int32_t path);

/* Debug: the kernel a decode step of `batch` rows would use under the current
 * path: *kind = 3 the row-split kernel, 2 the cluster kernel, 1 the
 * cooperative kernel (if it covers the shape; else the general sequence
 * runs), 0 the general sequence. Errors: FS_ERR_NULL, FS_ERR_INVALID. */
fs_status fs_debug_decode_kernel(const fs_model* model, int32_t batch, int32_t* kind);

/* Debug: dequantise Q8_0 blocks to fp32, out[n*k] = codes[n*k] * scales[n*(k/32)]
 * (all device, row-major). Bit-exact by construction. k % 32 == 0. */
fs_status fs_debug_dequant_q8_0(const int8_t* codes, const void* scales, int32_t n, int32_t k,
                                float* out, void* stream);

/* Debug: the model's last step on given rows: final RMSNorm of x (device fp32
 * [rows, H]), tied LM head, greedy choice. logits fp32 [rows, V] and argmax
 * int32 [rows] (device; either may be NULL). 1 <= rows <= 64. */
fs_status fs_debug_lm_head(fs_model* model, const float* x, int32_t rows, float* logits,
                           int32_t* argmax, void* stream);

/* Read and clear the model's device error word (waits for the device).
 * *code: 0 none, 1 a device token id was out of range, 2 a device-side
 * bounds check failed, 3 a cross-block wait gave up (timeout). */
fs_status fs_device_error(fs_model* model, int32_t* code);

/* Prefill GEMM operand precision. The tensor-core GEMMs of prefill take fp16
 * operands; with `split` = 1 each activation is carried as the sum of two fp16
 * terms (about 22 significant bits), which keeps prefill within 1e-3 of an
 * fp32 forward; `split` = 0 uses one fp16 term (faster, about 11 bits).
 * Default: 1. */
fs_status fs_set_prefill_split(fs_model* model, int32_t split);

/* The final RMSNorm + tied LM head + greedy selection of fs_debug_lm_head,
 * for callers that may not allocate device memory. The paper has no
 * counterpart: this is a deployment convenience, not a step of the method.
 *
 * Who it is for: callers that cannot call cudaMalloc — a host thread with a
 * latency budget (cudaMalloc can block on device-wide synchronisation and
 * driver locks), a process whose device memory is all reserved by another
 * framework's pool, or an embedding that lends us its buffers and forbids us
 * to own any. It needs no fs_model: pass the bf16 embedding [vocab, hidden]
 * (the tied LM head), the bf16 final-norm gains [hidden], and x, fp32
 * [rows, hidden] device rows. Outputs (device; either may be NULL, not both):
 * logits fp32 [rows, vocab], argmax int32 [rows] (lowest id on exact ties;
 * 0 if a row has no finite logit). Nothing is allocated: the normalised rows
 * and the per-block argmax partials live in one fixed 512 KiB array compiled
 * into the library, which every GPU that loads libfs holds until the process
 * exits. A call needs rows*hidden*4 (rounded up to 256) + rows*4*SMs*8 bytes
 * of it (148 SMs: 16 rows of hidden 1024 fit, 64 rows do not); larger calls
 * are rejected with FS_ERR_INVALID before anything runs.
 * Each call made outside a stream capture looks up the array's device
 * address afresh (so it stays right after cudaDeviceReset); a call captured
 * into a graph uses the address of the last uncaptured call on that device,
 * so make one uncaptured call (after any reset) before capturing. All calls
 * share the one array: two calls whose
 * work overlaps on the GPU (different streams, or different host threads on
 * one device) race on it and may return wrong results; serialise them.
 * Requirements: hidden % 64 == 0, 1 <= rows <= 64, rms_eps > 0, pointers
 * 16-byte aligned (argmax 4-byte). Errors: FS_ERR_NULL, FS_ERR_INVALID,
 * FS_ERR_ALIGN, FS_ERR_CUDA. */
fs_status fs_lm_head_argmax_noalloc(const void* embed, const void* final_norm, int32_t hidden,
                                    int32_t vocab, float rms_eps, const float* x, int32_t rows,
                                    float* logits, int32_t* argmax, void* stream);

/* Number of kernels libfs has launched in this process so far (all models,
 * all threads). For accounting in benchmarks; never reset. */
uint64_t fs_debug_kernel_launches(void);

/* Text of the last error raised on this thread ("" if none). */
const char* fs_last_error_string(void);

/* Name of a status code. */
const char* fs_status_string(fs_status status);

#ifdef __cplusplus
}
#endif

#endif /* FS_H */
