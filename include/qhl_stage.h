/*
 * qhl_stage.h - C ABI of the quantized hybrid layer-stage library (B200, sm_100a).
 *
 * A "stage" is a contiguous range of decoder layers of a hybrid Gated-DeltaNet +
 * attention model that a peer runs on the hidden state it is handed:
 *   - Unstable Legion: the peer-to-peer ChatGPT, "Splitting the workload": the
 *     model is cut into contiguous layer stages, and every stage holds the
 *     attention cache of its layers only.  "The runtime": a peer is handed an
 *     activation, pushes it through whatever layer range it was given, and
 *     hands the result on.
 *   - Peer-to-peer LLM inference in browser tabs, Qwen 3.8 27B (SwarmLLM
 *     README): peers hold layers 0-21 / 22-42 / 43-63 of a 64-layer model with a
 *     5,120-float hidden state, GGUF Q4_0 weights (4-bit values, one f16
 *     scale per block), prefill in 16-token batches, multi-token-prediction
 *     drafts checked together in one batched pass whose rejected tail is
 *     undone exactly in the recurrent state, and a speculative path that
 *     produces what plain decoding produces.
 *   - ChatTorrent README, "What it can run": the hybrid interleaves Gated
 *     DeltaNet layers and full-attention layers; the latter rotate only part
 *     of each head (partial RoPE), normalise q and k per head and gate their
 *     output; blocks use RMSNorm and SwiGLU; weights may be f32, f16 or q8.
 *
 * Each layer: h += mixer(RMSNorm1(h)); h += W_down(silu(W_gate x) * (W_up x)),
 * x = RMSNorm2(h).  Layer i is full attention iff i % attn_every == attn_every-1,
 * else gated DeltaNet.
 *
 * Conventions for every call:
 *   - All functions return a stage_status (0 = ok, negative = error); none
 *     throws, none aborts.  On error the stage's observable state (committed
 *     length, recurrent states, KV caches, pending pass) is unchanged and
 *     stage_last_error() describes the failure.
 *   - Device work is asynchronous and ordered on the CUDA stream given to
 *     stage_load.  Device-side faults of the stage's own kernels (a bounded
 *     wait that ran out) are reported by stage_sync().
 *   - A stage is not thread-safe; use one stage from one host thread at a time.
 */
#ifndef QHL_STAGE_H
#define QHL_STAGE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct stage stage_t;

typedef enum {
  STAGE_OK = 0,
  STAGE_E_ARG = -1,          /* null pointer, size or range out of bounds, unknown tensor name */
  STAGE_E_STATE = -2,        /* call not allowed now: pending pass, pos != committed length, nothing pending */
  STAGE_E_OOM = -3,          /* device memory allocation failed */
  STAGE_E_CUDA = -4,         /* a CUDA runtime call failed (message in stage_last_error) */
  STAGE_E_FORMAT = -5,       /* a required tensor is missing or has the wrong byte size */
  STAGE_E_UNSUPPORTED = -6,  /* shape the kernels do not implement */
  STAGE_E_DEVICE = -7        /* a stage kernel reported a device-side error (see stage_sync) */
} stage_status;

/* GGUF type ids of the supported block formats. */
typedef enum { STAGE_Q4_0 = 2, STAGE_Q8_0 = 8 } stage_qtype;

/* Model shape.  Supported: hidden, ffn multiples of 256; dn_dim == 128;
 * dn_v_heads a multiple of dn_k_heads; att_dim == 256; rope_dims == 64;
 * att_q_heads a multiple of att_kv_heads with att_q_heads/att_kv_heads <= 7;
 * 16 <= max_ctx <= 262144.  The 27B hybrid: 5120, 17408, 16, 48, 128, 24, 4, 256, 64,
 * 1e7, 1e-6, 4. */
typedef struct {
  int hidden;          /* H: width of the hidden state */
  int ffn;             /* F: SwiGLU intermediate width */
  int dn_k_heads;      /* DeltaNet key (and query) heads */
  int dn_v_heads;      /* DeltaNet value heads (state heads) */
  int dn_dim;          /* DeltaNet head dim (key and value) */
  int att_q_heads;     /* attention query heads */
  int att_kv_heads;    /* attention KV heads (GQA) */
  int att_dim;         /* attention head dim */
  int rope_dims;       /* leading head dims that RoPE rotates */
  double rope_theta;   /* RoPE base */
  float eps;           /* RMSNorm / QK-norm epsilon */
  int attn_every;      /* layer i is attention iff i % attn_every == attn_every - 1 */
  int max_ctx;         /* KV-cache rows per attention layer */
  int qtype;           /* STAGE_Q4_0 or STAGE_Q8_0 */
} stage_config;

/* One host tensor handed to stage_load.  The library reads `data` only during
 * the call (it is copied to the device and repacked); the caller keeps
 * ownership.  Names and contents, for each layer L of the range:
 *   "blk.L.norm1", "blk.L.norm2"            f32 [H]   RMSNorm weights
 *   DeltaNet layers:
 *     "blk.L.dn_in"   GGUF blocks [2*Hk*dk + Hv*dv + 2*Hv, H], rows q | k | v | b | a
 *     "blk.L.dn_out"  GGUF blocks [H, Hv*dv]
 *   attention layers:
 *     "blk.L.attn_in"     GGUF blocks [2*Hq*dh + 2*Hkv*dh, H], rows q | gate | k | v
 *     "blk.L.attn_q_norm", "blk.L.attn_k_norm"   f32 [dh]
 *     "blk.L.attn_out"    GGUF blocks [H, Hq*dh]
 *   "blk.L.ffn_gate", "blk.L.ffn_up"  GGUF blocks [F, H];  "blk.L.ffn_down"  GGUF blocks [H, F]
 * A GGUF matrix [rows, cols] is rows * cols/32 blocks in row-major block order;
 * Q4_0 block = binary16 d + 16 bytes (element j low nibble of byte j, element
 * j+16 high nibble, weight (nibble-8)*d); Q8_0 block = binary16 d + 32 int8
 * (weight q*d). */
typedef struct {
  const char* name;
  const void* data;
  size_t bytes;
} stage_tensor;

/* Create a stage for layers [layer_begin, layer_end) on the current CUDA
 * device.  A peer holds and runs one contiguous range of the model's layers
 * (Unstable Legion, "Splitting the workload"; SwarmLLM README, peer
 * diagram: layers 0-21 / 22-42 / 43-63), and its weights are GGUF blocks of
 * 4-bit values with an f16 scale (SwarmLLM README, paragraph after the peer
 * diagram, and model table: "GGUF Q4_0", "GGUF Q8_0 / Q4_0").  Uploads and repacks the weights, allocates recurrent states (zero),
 * KV caches (zero), a rollback ring of 17 snapshots per DeltaNet layer and all
 * scratch.  cuda_stream (a cudaStream_t, may be NULL for the legacy default
 * stream) orders every later call of this stage.  Blocks until the upload is
 * done.  On success *out owns all device memory until stage_free. */
stage_status stage_load(const stage_config* cfg, const stage_tensor* tensors, int n_tensors,
                        int layer_begin, int layer_end, void* cuda_stream, stage_t** out);

/* Run n_tok tokens (1..16) at positions pos .. pos+n_tok-1 through every layer
 * of the stage (one CUDA-graph launch).  The stage is handed an activation and
 * hands back the activation its layers produce (Unstable Legion, "The
 * runtime"); a token's pass reads every weight once, in one submission
 * (SwarmLLM README, paragraph after the peer diagram); prefill moves 16
 * tokens per hop and drafts are checked in one batched pass (SwarmLLM README,
 * feature list).  hidden_dev: caller-owned device f32
 * [n_tok, H], row-major, read and overwritten in place with the stage output.
 * pos must equal the committed length.  Leaves the pass pending: the next
 * forward is refused until stage_commit / stage_rollback.  Token t's output is
 * bit-identical to running the same tokens one at a time (forward(1) +
 * commit(1) each). */
stage_status stage_forward(stage_t* st, float* hidden_dev, int n_tok, int pos);

/* stage_forward from and to host memory, the whole round trip in one call:
 * hidden_in_host f32 [n_tok, H] is copied to the device, the pass runs, and
 * the result is copied to hidden_out_host f32 [n_tok, H] (both caller-owned,
 * row-major; they may be the same buffer).  All three steps are ordered on the
 * stage's stream: with page-locked buffers the call returns at once and
 * hidden_out_host is complete once that stream is synchronised (stage_sync);
 * with pageable buffers the CUDA runtime copies synchronously.  Same state
 * rules and errors as stage_forward; the output is bit-identical to it. */
stage_status stage_forward_host(stage_t* st, const float* hidden_in_host, float* hidden_out_host, int n_tok,
                                int pos);

/* stage_forward with the hidden state in IEEE binary16, the form a peer sends
 * on the wire (SwarmLLM README, paragraph under the benchmark table: one
 * token's 5,120-value hidden state is 10 KB as f16; github-Nehanth-swarmllm
 * summary, "How it works").  hidden_dev: caller-owned device binary16
 * [n_tok, H], row-major, 2-byte aligned, read and overwritten in place.  The
 * input is widened to f32 exactly, the pass is the one stage_forward runs, and
 * the output is its f32 result rounded to nearest even (magnitudes beyond
 * 65504 become +-inf, as IEEE rounding gives): for the same (f16) input
 * values, out_f16 == round_f16(out_f32 of stage_forward), bit for bit.
 * Same arguments, state rules and errors as stage_forward (STAGE_E_ARG also
 * for a misaligned pointer, before any device work). */
stage_status stage_forward_f16(stage_t* st, void* hidden_dev, int n_tok, int pos);

/* Prefill: run n_tok prompt tokens (1..16) at positions pos .. pos+n_tok-1
 * through every layer and commit them all in the same call (a prompt chunk is
 * never rolled back, so no per-token state snapshots are written: each
 * DeltaNet layer writes its final state only, 3.1 MB per layer instead of
 * n_tok times that).  Prefill sends 16 tokens per hop (SwarmLLM README,
 * feature list); the DeltaNet recurrence is what makes prefill serial and the
 * known gap (SwarmLLM README, under the benchmark table; github-Nehanth-
 * swarmllm summary, "How it works").  mode:
 *   STAGE_PREFILL_EXACT    the token-by-token recurrence, as stage_forward:
 *                          output and committed state bit-identical to
 *                          stage_forward + stage_commit(n_tok);
 *   STAGE_PREFILL_CHUNKED  the chunked closed form of the recurrence: per
 *                          value head one unit lower-triangular solve over the
 *                          chunk instead of n_tok dependent token steps, with
 *                          every dot product against the starting state
 *                          independent; within rounding of the exact mode, not
 *                          bit-identical to it.
 * hidden_dev as in stage_forward (read and overwritten in place); pos must
 * equal the committed length; no pass may be pending; afterwards the committed
 * length is pos + n_tok and nothing is pending. */
typedef enum { STAGE_PREFILL_EXACT = 0, STAGE_PREFILL_CHUNKED = 1 } stage_prefill_mode;
stage_status stage_prefill(stage_t* st, float* hidden_dev, int n_tok, int pos, int mode);

/* Keep the first n_accepted tokens (0..n_tok) of the pending pass: the
 * accepted prefix of a speculative batch, whose rejected tail is undone
 * exactly in the recurrent state (SwarmLLM README, paragraph after the peer
 * diagram; github-Nehanth-swarmllm summary, "How it works").  Each
 * DeltaNet state becomes the snapshot after token n_accepted (no copy: the
 * ring index moves) and the committed length becomes pos + n_accepted.  KV
 * rows beyond it stay in memory but are never read and are overwritten by the
 * next pass.  The result is bit-identical to having run only those tokens. */
stage_status stage_commit(stage_t* st, int n_accepted);

/* Discard the pending pass: identical to stage_commit(st, 0).  This is the
 * exact rollback of the recurrent state and KV cache when no draft is
 * accepted (SwarmLLM README, paragraph after the peer diagram). */
stage_status stage_rollback(stage_t* st);

/* Start a new sequence: zero every recurrent state, committed length 0.
 * Refused while a pass is pending. */
stage_status stage_reset(stage_t* st);

/* Wait for the stage's stream; returns STAGE_E_DEVICE if a stage kernel
 * reported a device-side error since the last stage_sync (and clears it). */
stage_status stage_sync(stage_t* st);

/* Committed length (positions in the KV caches that are part of the sequence). */
int stage_committed_len(const stage_t* st);

/* Number of tokens of the pending pass, 0 if none. */
int stage_pending(const stage_t* st);

/* Copy the current state of DeltaNet layer `layer` (absolute index) to/from
 * host memory: f32 [Hv, dv, dk] row-major (S[h][i][j], i the value dim), bytes
 * must be Hv*dv*dk*4.  Synchronous.  Refused while a pass is pending. */
stage_status stage_get_dn_state(stage_t* st, int layer, float* host_dst, size_t bytes);
stage_status stage_set_dn_state(stage_t* st, int layer, const float* host_src, size_t bytes);

/* Copy the KV cache of attention layer `layer` to/from host memory: binary16
 * bit patterns [Hkv, max_ctx, dh] for K and for V, bytes_each =
 * Hkv*max_ctx*dh*2.  Synchronous.  Refused while a pass is pending. */
stage_status stage_get_kv(stage_t* st, int layer, uint16_t* k_host, uint16_t* v_host, size_t bytes_each);
stage_status stage_set_kv(stage_t* st, int layer, const uint16_t* k_host, const uint16_t* v_host,
                          size_t bytes_each);

/* Set the committed length (e.g. after filling the KV caches with stage_set_kv).
 * 0 <= kv_len <= max_ctx - 1.  Refused while a pass is pending. */
stage_status stage_set_kv_len(stage_t* st, int kv_len);

/* Dequantise row `row` of weight tensor `tensor` (a name as in stage_tensor)
 * from the stage's packed device copy, with the same device code the GEMV
 * uses, into host_dst (f32 [cols], the tensor's column count; dst_elems = the
 * buffer's capacity in floats, STAGE_E_ARG if it is smaller, before any
 * device work).  Synchronous.  Used to check that the repacked weights
 * dequantise bit-exactly. */
stage_status stage_debug_dequant(stage_t* st, const char* tensor, int row, float* host_dst, size_t dst_elems);

/* How a forward pass runs on the device.
 *   STAGE_PASS_KERNELS (default): one kernel per step (stage input, then per
 *     layer in-projection, mixer, out-projection, gate/up, down), recorded in
 *     a CUDA graph, each a programmatic dependent of the one before.
 *   STAGE_PASS_PERSISTENT: one cooperative kernel of one CTA per SM runs the
 *     whole pass, its phases separated by a grid-wide arrival counter; its
 *     producer streams every projection's weights across phase boundaries.
 *     Used for n_tok 1..4 when the mixers' scratch fits (attention context of
 *     at most ~3400 chunks of 64 rows); other passes and prefill run as
 *     kernels.
 * Both run the same units with the same split and reduction order, so they
 * give bit-identical results.  Refused while a pass is pending; waits for the
 * stage's stream and drops the recorded graphs. */
typedef enum { STAGE_PASS_KERNELS = 0, STAGE_PASS_PERSISTENT = 1 } stage_pass_mode;
stage_status stage_set_pass_mode(stage_t* st, int mode);

/* 1 if an n_tok-token forward would run as the persistent kernel, 0 if as a
 * chain of kernels, -1 for a NULL stage or n_tok outside 1..16. */
int stage_pass_persistent(stage_t* st, int n_tok);

/* Failure injection for tests of the device-side error path (no counterpart
 * on the pages; the stage's kernels bound every wait, and this makes one run
 * out without faulting anything).  fault_item >= 0: in the next recorded
 * passes, CTA 0 of the first layer's in-projection never requests the quants
 * of its local item fault_item, so the wait for them runs out; -1 turns that
 * off.  wait_limit: iteration cap of every bounded wait of the stage's GEMV
 * kernels (0 = the default, seconds; a test passes a few thousand so the
 * injected stall ends in milliseconds).  The pass then finishes with garbage
 * in its outputs and stage_sync() returns STAGE_E_DEVICE (clearing the error
 * word and the stream-K tile counters); stage_rollback() keeps the committed
 * state intact, so the next pass is correct once injection is off again.
 * Drops the recorded graphs; refused while a pass is pending. */
stage_status stage_debug_inject(stage_t* st, int fault_item, unsigned wait_limit);

/* Bytes of weight storage the stage streams per pass (packed quants + scales). */
size_t stage_weight_bytes(const stage_t* st);

/* Human-readable description of the last error of this stage ("" if none). */
const char* stage_last_error(const stage_t* st);

/* Free all device memory of the stage (waits for its stream).  NULL is a no-op. */
void stage_free(stage_t* st);

/* ---------------------------------------------------------------------------
 * Kernel-level entry points (one hot-path kernel each, no stage object).
 * Pointers named *_dev are device memory owned by the caller; the call is
 * asynchronous on `stream`.  Return 0 on success or a negative stage_status;
 * qhl_last_error() gives the message (per host thread).
 * ------------------------------------------------------------------------- */

/* Bytes of the packed (repacked) form of a GGUF matrix [rows, cols]:
 * ceil(rows/128) * cols/256 items of 18432 (Q4_0) or 34816 (Q8_0) bytes.
 * For a gate/up pair (paired != 0) rows is the number of features of each
 * matrix and the result holds both: ceil(rows/64) items per 256 columns.
 * Returns 0 for an unsupported shape (cols % 256 != 0, rows <= 0). */
size_t qhl_packed_bytes(int qtype, int rows, int cols, int paired);

/* Repack GGUF blocks (device, [rows, cols/32] blocks) into the packed layout
 * the GEMV streams.  gguf_b_dev: second matrix of a gate/up pair (its rows are
 * interleaved tile by tile with gguf_dev's for the SwiGLU epilogue), or NULL.
 * packed_dev must hold qhl_packed_bytes(qtype, rows, cols, gguf_b_dev != NULL)
 * bytes and be 16-byte aligned. */
int qhl_repack(int qtype, int rows, int cols, const void* gguf_dev, const void* gguf_b_dev,
               void* packed_dev, void* stream);

/* Dequantise rows [row0, row0+nrows) of a packed matrix into out_dev (f32
 * [nrows, cols]) with the GEMV's own conversion code; bit-exact by design.
 * packed_dev must be 16-byte aligned (STAGE_E_ARG otherwise).
 * paired != 0: rows 0..rows-1 address the first matrix of a pair, rows
 * rows..2*rows-1 the second. */
int qhl_dequant(int qtype, int rows, int cols, const void* packed_dev, int paired, int row0, int nrows,
                float* out_dev, void* stream);

/* y = x W^T for n_tok tokens (1..16): x_dev f32 [n_tok, cols], y_dev f32
 * [n_tok, rows], W packed (not paired).  Reduction order is fixed and
 * independent of n_tok (a batched call equals n_tok single calls bit for bit).
 * At most 2^31 - 1 packed items (ceil(rows/128) * cols/256), else STAGE_E_ARG.
 * Uses library-owned scratch (stream-K partials and tile counters, allocated
 * on first use per device and grown on demand); concurrent calls on different
 * streams of the same device must not overlap. */
int qhl_qgemv(int qtype, int rows, int cols, const void* packed_dev, const float* x_dev, int n_tok,
              float* y_dev, void* stream);

/* n_tok sequential gated-DeltaNet steps (dn_dim 128) for all Hv value heads.
 * y_dev: f32 [n_tok, 2*Hk*128 + Hv*128 + 2*Hv] raw in-projection rows
 * q | k | v | b | a per token (q, k are L2-normalised here; beta = sigmoid(b),
 * alpha = exp(-softplus(a))).  s_in_dev: f32 [Hv, 128, 128] state before the
 * first token (not modified).  snaps_dev: f32 [n_tok, Hv, 128, 128] receives
 * the state after each token.  o_dev: f32 [n_tok, Hv*128] receives o_t = S_t q_t.
 * y_dev, s_in_dev and snaps_dev are read / written as 16-byte vectors and must
 * be 16-byte aligned (STAGE_E_ARG otherwise, before any device work). */
int qhl_deltanet_step(int Hk, int Hv, const float* y_dev, int n_tok, const float* s_in_dev,
                      float* snaps_dev, float* o_dev, void* stream);

/* The GEMV of qhl_qgemv for callers that cannot allocate device memory at
 * call time: a process whose memory pool already owns the whole GPU, or a
 * latency-critical loop that must not pay for cudaMalloc / cudaFree (which can
 * synchronise the device).  The pages have no counterpart of this call; it
 * exists for such callers only.  Same arguments and results as qhl_qgemv (same
 * kernels, so the outputs are identical), but every piece of scratch lives in
 * one static device array of about 4.8 MiB that each GPU loading this library
 * holds until the process exits; the call itself allocates nothing.  Limits:
 * n_tok * (cols / 256) * 2048 bytes must not exceed 2.25 MiB (for example cols
 * up to 18432 at 16 tokens, 294912 at 1 token), rows at most 2097152, and the
 * device at most 160 SMs; larger problems return STAGE_E_ARG
 * (STAGE_E_UNSUPPORTED for the SM count) before any device work.  The first call on a device looks up
 * the array's device address and sets kernel attributes; make that first call
 * before any stream capture.  All calls share the one array, which keeps the
 * last call's contents (the tile counters are cleared by every call): calls
 * that overlap on the GPU, e.g. on two streams of the same device, race and
 * must be serialised by the caller. */
int qhl_qgemv_noalloc(int qtype, int rows, int cols, const void* packed_dev, const float* x_dev, int n_tok,
                      float* y_dev, void* stream);

/* Wait for `stream`, then report and clear the device-side error word of the
 * qhl_qgemv / qhl_qgemv_noalloc kernels on the current device: STAGE_E_DEVICE
 * if one of their bounded waits ran out since the last qhl_sync (their output
 * is then garbage; the tile counters are cleared with the word so that later
 * calls are correct), 0 otherwise.  Allocates nothing. */
int qhl_sync(void* stream);

/* Failure injection for tests of that error path (no counterpart on the
 * pages): later qhl_qgemv calls make CTA 0 skip the quants of its local item
 * fault_item (-1: off) and cap every bounded wait at wait_limit iterations
 * (0: the default), so one wait runs out without faulting anything.
 * Process-wide; qhl_qgemv_noalloc is not affected. */
int qhl_debug_inject(int fault_item, unsigned wait_limit);

/* Message of the last failed qhl_* call on this host thread ("" if none). */
const char* qhl_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* QHL_STAGE_H */
