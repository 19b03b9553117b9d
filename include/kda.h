/*
 * kda.h — C ABI of libkda.so, a B200 (sm_100a) implementation of the Kimi Delta
 * Attention (KDA) token mixer.
 *
 * The operation (page "Ling-3.0-flash: a 124B open MoE that runs like a 5B and
 * reaches for 1M tokens", section "KDA: constant-size memory over a very long
 * context"): a gated delta-rule linear attention that keeps one fixed d_k x d_v
 * state S per head. Each token decays S per key channel (alpha_t, the erase),
 * then writes the key/value association with the delta rule (beta_t k_t v_t^T),
 * and the query reads the state. The displayed equation is missing from that
 * page; the library implements
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t                      alpha_t = exp(log_alpha_t) per key channel
 *
 * Head geometry of the model (page "Ling 3.0 Flash", table "Every architecture
 * field"): 32 key heads = 32 value heads, head dim 128, short-conv kernel 4.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named "device" are CUDA device memory owned by the caller; the
 *   library never frees or retains them past the call. Nothing persistent is
 *   allocated: scratch comes from the caller's `workspace`.
 * - Layouts are row-major, last index fastest, token-major packed:
 *     q, k, log_alpha   [total_T, H, dk]      v, out, gate   [total_T, H, dv]
 *     beta              [total_T, H]          states         [N, H, dk, dv]
 *   Fixed-length batches B x T are the same memory with total_T = B*T, N = B.
 * - Sequences: `cu_seqlens` is a device int32 array [N+1] with cu[0] = 0,
 *   cu[N] = total_T and cu[n] <= cu[n+1] (zero-length sequences allowed). NULL
 *   means N equal sequences of total_T / N tokens.
 * - No query scale is applied (o is linear in q: pre-scale q if wanted).
 * - All calls are asynchronous on `stream` (0 = legacy default stream). Argument
 *   checks are synchronous on the host and return before any launch. A launch
 *   failure returns KDA_ERR_CUDA. The library never aborts, traps or prints.
 * - Problems that only the device can see (a cu_seqlens that is not
 *   non-decreasing or overruns total_T; a wait inside a kernel that ran out of
 *   time) set bits in a status word held in `workspace`; the outputs are then
 *   unspecified (a bad cu_seqlens may leave every sequence unwritten). Read the
 *   word with kda_workspace_status() after the stream has run the call.
 * - Thread safety: calls may be issued from several host threads; the message
 *   returned by kda_last_error() is thread-local.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* kda_stream_t; /* same object as cudaStream_t */

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1, /* NULL pointer, bad size, dtype, or misalignment   */
  KDA_ERR_UNSUPPORTED = 2, /* valid request outside what this build implements  */
  KDA_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than the query returned  */
  KDA_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed        */
  KDA_ERR_RANGE = 5        /* device-detected range violation (status word set)  */
} kda_status;

typedef enum { KDA_DT_F32 = 0, KDA_DT_BF16 = 1 } kda_dtype;

/* Bits of the device status word (kda_workspace_status). */
#define KDA_DEVFLAG_BAD_SEQLENS 0x1u  /* cu_seqlens not monotone / out of range */
#define KDA_DEVFLAG_DECAY_RANGE 0x2u  /* reserved, never set: every decay is in range (the
                                         prefill walks chunks of very strong decay token by
                                         token, see kda_chunk_fwd)                          */
#define KDA_DEVFLAG_BAD_INDEX 0x4u    /* a state index outside [0, pool_size)    */
#define KDA_DEVFLAG_WAIT_TIMEOUT 0x80000000u /* a wait inside a kernel gave up after 2 s (a lost
                                         arrival); the kernel returned early, outputs
                                         unspecified, the CUDA context stays usable         */

/* Largest head dimensions this build accepts (d_k, d_v <= 128; the model uses 128). */
#define KDA_MAX_HEAD_DIM 128

/* Human-readable name of a status code (static string). */
KDA_API const char* kda_status_string(kda_status s);

/* Detail of the last non-OK status returned on this host thread ("" if none). */
KDA_API const char* kda_last_error(void);

/* Library version, "major.minor.patch". */
KDA_API const char* kda_version(void);

/*
 * Workspace, in bytes, that kda_chunk_fwd needs for these sizes (a multiple of
 * 256; never 0, the status word always lives there). Returns 0 for sizes the
 * library rejects.
 *
 * Beyond the status word (and, for head dims below 128, zero-padded copies of
 * the inputs), the workspace holds the scratch of the two-pass prefill: about
 * 145 KB per (64-token chunk, head), e.g. 303 MB for one 4096-token sequence of
 * 32 heads. The two-pass form is used for at most 74 (sequence, head) pairs
 * (N * H <= 74) and at most 32 GiB of scratch; otherwise the call runs a
 * single-pass kernel that needs no scratch and the query leaves it out.
 */
KDA_API size_t kda_chunk_fwd_workspace(int64_t total_T, int N, int H, int dk, int dv, kda_dtype qkv_dtype);

/*
 * Chunked prefill: runs the recurrence above over every packed sequence.
 *
 * Defining passage: the KDA section cited at the top (the gated decay, the
 * delta-rule write, the read with the query, a state whose size does not
 * depend on T). The chunk-parallel form used on the device (64-token chunks,
 * the WY/UT triangular solve, tensor-core GEMMs, fp32 state carried between
 * chunks) computes the same result up to rounding.
 *
 *   q, k       device, [total_T, H, dk], dtype qkv_dtype (bf16 or fp32)
 *   v          device, [total_T, H, dv], dtype qkv_dtype
 *   log_alpha  device fp32 [total_T, H, dk]: natural log of the per-channel
 *              decay, <= 0 (finite). Any decay is supported. A 64-token chunk
 *              (aligned to the sequence start) whose decay summed over its tokens
 *              stays within 20 nats in every key channel takes the tensor-core form,
 *              which multiplies k e^g by k e^-g; any other chunk is walked token by
 *              token with the recurrence itself (exact for any decay, slower).
 *   beta       device fp32 [total_T, H], the write strength (sigmoid output).
 *   initial_state  device fp32 [N, H, dk, dv] or NULL (zero state).
 *   cu_seqlens device int32 [N+1] or NULL (equal lengths; total_T % N == 0).
 *   out        device [total_T, H, dv], dtype qkv_dtype; rows of zero-length
 *              sequences are not written.
 *   final_state device fp32 [N, H, dk, dv] or NULL (not written). It may alias
 *              initial_state exactly (same pointer); partial overlap is an error.
 *   workspace  device, >= kda_chunk_fwd_workspace(...) bytes, 256-byte aligned;
 *              its contents on entry are ignored.
 *
 * Alignment: every tensor pointer must be 16-byte aligned. Returns KDA_OK once
 * the work is enqueued.
 */
KDA_API kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, kda_dtype qkv_dtype,
                         const float* log_alpha, const float* beta, const float* initial_state,
                         const int32_t* cu_seqlens, int64_t total_T, int N, int H, int dk, int dv,
                         void* out, float* final_state, void* workspace, size_t workspace_bytes,
                         kda_stream_t stream);

/*
 * Decode step: one token per (sequence, head), state updated in place.
 *
 * Defining passage: the same KDA section (each token updates the fixed-size
 * state in place; decode does not grow with context). Per (n, h):
 *     S' = Diag(exp(log_alpha)) S;  u = beta (v - S'^T k);  S <- S' + k u^T;
 *     out = S^T q  (= S'^T q + u (k . q)).
 *
 *   q, k       device [N, H, dk], dtype qkv_dtype;  v device [N, H, dv]
 *   log_alpha  device fp32 [N, H, dk];  beta device fp32 [N, H]
 *   state      device fp32 [N, H, dk, dv], read and overwritten in place
 *   out        device [N, H, dv], dtype qkv_dtype; must not overlap state
 * Alignment: state and out 16-byte aligned; other pointers 4-byte aligned.
 */
KDA_API kda_status kda_decode_step(const void* q, const void* k, const void* v, kda_dtype qkv_dtype,
                           const float* log_alpha, const float* beta, float* state,
                           int N, int H, int dk, int dv, void* out, kda_stream_t stream);

/*
 * Serving decode step of the full mixer: one new token for each of N sequences,
 * through the same steps as kda_mixer_fwd — conv4 on q, k, v (over the sequence's
 * last three raw inputs and this token), L2 norm of q and k, the KDA decode step,
 * the sigmoid output gate — with the states and the conv histories kept in pools
 * indexed per sequence (the KDA panel of the article cited above, one token at a
 * time; the pool indexing is the library's own serving layout).
 *
 *   q_raw, k_raw, v_raw  device bf16 [N, H, d]: this token's raw projections
 *   conv_w       device fp32 [3, H*d, 4] (q, k, v), as for kda_mixer_fwd
 *   log_alpha    device fp32 [N, H, d];  beta device fp32 [N, H]
 *   gate         device bf16 [N, H, d] or NULL (no gate)
 *   state_pool   device fp32 [pool_size, H, d, d], read and updated in place
 *   conv_pool    device bf16 [pool_size, H, 3, 3, d]: per slot and head, for q, k, v
 *                the last three raw rows, oldest first; updated in place (the
 *                oldest row drops, this token's row is appended). A new sequence
 *                starts from zeros; after a prefill it holds the prompt's last three
 *                raw q, k, v rows (zeros where the prompt is shorter).
 *   state_indices device int32 [N]: the slot of each sequence, or NULL for slot n.
 *                Slots must be distinct within a call (two sequences on one slot
 *                race); an index outside [0, pool_size) leaves that sequence untouched
 *                and sets KDA_DEVFLAG_BAD_INDEX in `status`.
 *   out          device bf16 [N, H, d]
 *   status       device uint32 word (e.g. a workspace's first word) or NULL; read it
 *                with kda_workspace_status.
 * Requires dk = dv = d = 128. Alignment: 16 bytes for every pointer but
 * state_indices (4). Returns KDA_OK once the work is enqueued.
 */
KDA_API kda_status kda_mixer_decode_step(const void* q_raw, const void* k_raw, const void* v_raw,
                                 const float* conv_w, const float* log_alpha, const float* beta,
                                 const void* gate, float* state_pool, void* conv_pool,
                                 const int32_t* state_indices, int pool_size, int N, int H, int dk, int dv,
                                 void* out, void* status, kda_stream_t stream);

/*
 * K consecutive tokens per sequence through the serving decode step (speculative
 * decoding: K draft tokens in one call). Same arguments as kda_mixer_decode_step with
 * a token axis: q_raw, k_raw, v_raw, log_alpha, gate, out [N, K, H, d]; beta [N, K, H].
 * The state of a (sequence, head) stays on chip across the K tokens, so a call moves
 * it once instead of K times.
 *   state_ckpt  device fp32 [N, K, H, d, d] or NULL
 *   conv_ckpt   device bf16 [N, K, H, 3, 3, d] or NULL (both or neither)
 * Without checkpoints the pools receive the state and history after the K tokens.
 * With checkpoints the pools are left unchanged and entry j holds the state and
 * history after token j; kda_mixer_decode_commit then installs the entry of the last
 * accepted token. K = 1 without checkpoints is kda_mixer_decode_step.
 */
KDA_API kda_status kda_mixer_decode_tokens(const void* q_raw, const void* k_raw, const void* v_raw,
                                   const float* conv_w, const float* log_alpha, const float* beta,
                                   const void* gate, float* state_pool, void* conv_pool,
                                   const int32_t* state_indices, int pool_size, int N, int K, int H, int dk,
                                   int dv, void* out, float* state_ckpt, void* conv_ckpt, void* status,
                                   kda_stream_t stream);

/*
 * After kda_mixer_decode_tokens with checkpoints: for each sequence n with
 * accepted[n] = a (device int32 [N], 0 <= a <= K) copy checkpoint a - 1 into the
 * sequence's pool slot (a = 0 keeps the slot as it was before the K tokens). An
 * out-of-range slot or count sets KDA_DEVFLAG_BAD_INDEX in `status` and leaves that
 * sequence untouched. d = 128; pointers 16-byte aligned (accepted, state_indices: 4).
 */
KDA_API kda_status kda_mixer_decode_commit(const float* state_ckpt, const void* conv_ckpt,
                                   const int32_t* accepted, float* state_pool, void* conv_pool,
                                   const int32_t* state_indices, int pool_size, int N, int K, int H, int d,
                                   void* status, kda_stream_t stream);

/*
 * Affine map of states: out[i] = M[i] S[i] + B[i] for `count` d x d fp32 matrices
 * (row-major, M acting on the key rows). The state after a stretch of tokens is
 * affine in the state before it (same KDA section): S_end = M S_start + B, where M
 * is the stretch's final state from the identity with zero values and B its final
 * state from zero. Composing the maps of consecutive segments gives each segment
 * its starting state, which lets one long sequence be prefilled in parallel across
 * devices (context parallelism; see gated_delta_rule_137_b200.context_parallel).
 *   M      device fp32 [count, d, d]
 *   S, B   device fp32 [count, d, d] or NULL (zero)
 *   out    device fp32 [count, d, d]; may be B (in-place add), not M or S
 * d must be 128; pointers 16-byte aligned.
 */
KDA_API kda_status kda_state_affine(const float* M, const float* S, const float* B, float* out, int64_t count,
                            int d, kda_stream_t stream);

/*
 * Segment maps, for prefilling one long sequence on several devices at once (context
 * parallelism). The state after a stretch of tokens is affine in the state before it
 * (the KDA section cited at the top: each token multiplies the state on the left by
 * (I - beta k k^T) Diag(alpha) and adds beta k v^T), so a segment acts on the state as
 * S_end = M S_start + B: M is the segment's final state from the identity with zero
 * values, B its final state from zero. kda_segment_maps computes both from one pass over
 * the segment's chunks and keeps that pass's per-chunk operands in `workspace`;
 * kda_segment_prefill then runs the segment from any start state on those operands (once
 * the start state is known, e.g. after the ranks have exchanged their maps and folded the
 * earlier segments' maps with kda_state_affine). Together they cost about one prefill and
 * a half instead of three.
 *
 *   q, k, v, qkv_dtype, log_alpha, beta, cu_seqlens, total_T, N, H: as for kda_chunk_fwd
 *              (dk = dv = 128; total_T >= 1)
 *   M, B       device fp32 [N, H, 128, 128], written
 *   workspace  device, >= kda_segment_maps_workspace(...) bytes, 16-byte aligned; keep it
 *              untouched between the two calls (its status word holds the flags of both)
 * kda_segment_prefill writes out ([total_T, H, 128], qkv_dtype) and final_state (fp32
 * [N, H, 128, 128] or NULL) from initial_state (fp32 [N, H, 128, 128] or NULL: zero), for
 * the same segment (same sizes and cu_seqlens as the maps call). Status words and errors
 * as for kda_chunk_fwd.
 */
KDA_API size_t kda_segment_maps_workspace(int64_t total_T, int N, int H, int dk, int dv);
KDA_API kda_status kda_segment_maps(const void* q, const void* k, const void* v, kda_dtype qkv_dtype,
                                    const float* log_alpha, const float* beta, const int32_t* cu_seqlens,
                                    int64_t total_T, int N, int H, int dk, int dv, float* M, float* B,
                                    void* workspace, size_t workspace_bytes, kda_stream_t stream);
KDA_API kda_status kda_segment_prefill(void* workspace, size_t workspace_bytes, kda_dtype qkv_dtype,
                                       const float* initial_state, const int32_t* cu_seqlens, int64_t total_T,
                                       int N, int H, int dk, int dv, void* out, float* final_state,
                                       kda_stream_t stream);

/*
 * A chain of affine maps in one call: S <- M_j S + B_j for j = 0 .. maps-1, starting from
 * S0 (NULL: zero); out receives the result. The start state of segment r of a context-
 * parallel prefill is the fold of the maps of segments 0 .. r-1 (see kda_segment_maps).
 *   MB   device fp32 [maps, 2, count, d, d]: M then B of each map (the layout of the
 *        ranks' all-gathered maps)
 *   S0   device fp32 [count, d, d] or NULL;  out device fp32 [count, d, d] (may be S0)
 * d must be 128; pointers 16-byte aligned; fp32 arithmetic.
 */
KDA_API kda_status kda_state_fold(const float* MB, int maps, const float* S0, float* out, int64_t count, int d,
                                  kda_stream_t stream);

/* Workspace for kda_mixer_fwd (bytes, multiple of 256; 0 for rejected sizes): the
 * status word plus the two-pass prefill's scratch, sized as for kda_chunk_fwd (the
 * conv/L2 stage runs inside the prefill's first pass and needs no buffer of its own). */
KDA_API size_t kda_mixer_fwd_workspace(int64_t total_T, int N, int H, int dk, int dv);

/*
 * Full mixer prefill: the KDA panel of the same article — q and k pass through
 * a short causal depthwise conv and an L2 norm, v through a conv, then the KDA
 * recurrence, then a sigmoid output gate.
 *   conv (kernel 4, page "Ling 3.0 Flash", field short_conv_kernel_size):
 *     y[t, c] = sum_{j=0..3} w[c, j] x[t-3+j, c], zero history at each sequence
 *     start, no bias, identity activation;
 *   L2 norm per (token, head) of q and k: x / sqrt(sum x^2 + 1e-6), in fp32;
 *   gate: out = o * sigmoid(g) (skipped when gate is NULL).
 *
 *   q_raw, k_raw  device bf16 [total_T, H, dk];  v_raw device bf16 [total_T, H, dv]
 *   conv_w        device fp32 [3, H*d, 4] (q, k, v weights; requires dk == dv = d)
 *   gate          device bf16 [total_T, H, dv] or NULL
 *   log_alpha, beta, initial_state, cu_seqlens, out (bf16), final_state,
 *   workspace, stream: as for kda_chunk_fwd.
 */
KDA_API kda_status kda_mixer_fwd(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                         const float* log_alpha, const float* beta, const void* gate,
                         const float* initial_state, const int32_t* cu_seqlens, int64_t total_T,
                         int N, int H, int dk, int dv, void* out, float* final_state,
                         void* workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * Full mixer prefill that hands its sequences over to the serving decode
 * (kda_mixer_decode_step / kda_mixer_decode_tokens): the same computation as
 * kda_mixer_fwd, but each sequence's final state goes into its slot of state_pool, and
 * its last three raw q, k, v rows (oldest first, zeros where the prompt is shorter) into
 * the same slot of conv_pool, the layout the decode step reads. Each sequence starts
 * with a zero conv history (a new prompt) and from initial_state[n] (or zero).
 *   state_pool    device fp32 [pool_size, H, d, d]; slots no sequence names are untouched
 *   conv_pool     device bf16 [pool_size, H, 3, 3, d]
 *   state_indices device int32 [N]: the slot of each sequence, or NULL for slot n (then
 *                 pool_size >= N). Slots must be distinct within a call. A slot outside
 *                 [0, pool_size) sets KDA_DEVFLAG_BAD_INDEX; that sequence's out rows are
 *                 still written, its pools are not.
 *   the other arguments and the workspace (kda_mixer_fwd_workspace): as for kda_mixer_fwd.
 * initial_state, state_pool, conv_pool and out must not overlap. Requires dk = dv = d = 128.
 * (The article's deployment runs prefill and decode on one cache of states; the pooled
 * layout and this hand-off are the library's own.)
 */
KDA_API kda_status kda_mixer_fwd_pooled(const void* q_raw, const void* k_raw, const void* v_raw,
                                        const float* conv_w, const float* log_alpha, const float* beta,
                                        const void* gate, const float* initial_state, const int32_t* cu_seqlens,
                                        int64_t total_T, int N, int H, int dk, int dv, void* out,
                                        float* state_pool, void* conv_pool, const int32_t* state_indices,
                                        int pool_size, void* workspace, size_t workspace_bytes,
                                        kda_stream_t stream);

/*
 * Full mixer prefill with the decay gate made from its pre-activation (the article's
 * KDA panel names a softplus for the gate; the form read here is one positive scale
 * per head): log_alpha = -a_scale[h] * softplus(a_pre), computed in fp32 as the
 * pre-activation is read, so the gate costs 2 bytes per channel instead of 4.
 * Arguments as kda_mixer_fwd, with log_alpha replaced by
 *   a_pre    device bf16 [total_T, H, dk]
 *   a_scale  device fp32 [H], > 0
 * and the workspace sized by kda_mixer_fwd_gate_workspace (this entry point always
 * runs the two-pass prefill; 0 from the query means the sizes are too large for it).
 */
KDA_API size_t kda_mixer_fwd_gate_workspace(int64_t total_T, int N, int H, int dk, int dv);
KDA_API kda_status kda_mixer_fwd_gate(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                              const void* a_pre, const float* a_scale, const float* beta, const void* gate,
                              const float* initial_state, const int32_t* cu_seqlens, int64_t total_T,
                              int N, int H, int dk, int dv, void* out, float* final_state,
                              void* workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * Full mixer prefill without a workspace, for callers that cannot allocate device
 * memory where they run the mixer (a plugin whose host framework owns every device
 * allocation, a serving loop that may not call cudaMalloc). The paper has no
 * counterpart: it takes kda_mixer_fwd's arguments minus the workspace and runs the
 * mixer in two stages (conv/L2 into fp32 scratch, then the recurrence); results
 * match kda_mixer_fwd within the parity tolerance.
 *
 * Scratch is a fixed array in the library's device memory (about 24 MiB per GPU
 * that loads the library, held until the process exits). Limit: total_T * H <=
 * 16384 token-heads; larger calls return KDA_ERR_UNSUPPORTED before any launch.
 * The first call on a device looks the array up (cudaGetSymbolAddress) with that
 * device current; make it before any stream capture. With CUDA's lazy module
 * loading (the default) that first call is also when the driver loads the
 * library's device code and reserves the array, so a device that is already full
 * can fail it with KDA_ERR_CUDA: make one warm-up call (total_T = N = 0 does the set-up
 * and launches nothing) while memory is free. All calls on a device share the
 * array, which keeps the last call's contents (the status word is cleared at the
 * start of each call); calls that overlap on the GPU race and give undefined
 * results. Allocates nothing.
 */
KDA_API kda_status kda_mixer_fwd_noalloc(const void* q_raw, const void* k_raw, const void* v_raw,
                                         const float* conv_w, const float* log_alpha, const float* beta,
                                         const void* gate, const float* initial_state, const int32_t* cu_seqlens,
                                         int64_t total_T, int N, int H, int dk, int dv, void* out,
                                         float* final_state, kda_stream_t stream);

/*
 * The device status word of kda_mixer_fwd_noalloc (it lives in the same static array
 * on the current device): synchronises `stream`, copies the word to the host, clears
 * it. Returns KDA_ERR_RANGE when any KDA_DEVFLAG_* bit was set (e.g. a bad
 * cu_seqlens in the last call), KDA_OK otherwise; *flags (if not NULL) receives the
 * bits. Allocates nothing; the same set-up rule as kda_mixer_fwd_noalloc applies.
 */
KDA_API kda_status kda_mixer_fwd_noalloc_status(kda_stream_t stream, uint32_t* flags);

/*
 * Workspace for kda_chunk_bwd (bytes, multiple of 256; 0 for rejected sizes): the
 * status word and a checkpoint of the state every 8 tokens (64 KB per 8 tokens and
 * head, e.g. 1.09 GB for one 4096-token sequence of 32 heads).
 */
KDA_API size_t kda_chunk_bwd_workspace(int64_t total_T, int N, int H, int dk, int dv);

/*
 * Backward of the recurrence (training): given the gradient of the loss with respect
 * to the outputs (and optionally the final state), the gradients with respect to every
 * input of kda_chunk_fwd. Defining passage: the same KDA section; the gradient is that
 * of the token recurrence, which the chunked forward computes up to rounding. Writing
 * one token with P = Diag(alpha) S_prev, w = P^T k, u = beta (v - w), S = P + k u^T,
 * o = S^T q and walking the tokens backwards with G the gradient of S:
 *     G += q do^T;  dq = S do;  du = G^T k;  dv = beta du;  dbeta = du . (v - w);
 *     dk = G u - beta P du;  dP = G - beta k du^T;
 *     dlog_alpha_i = sum_j dP_ij P_ij;  G <- Diag(alpha) dP.
 * The states are recomputed from checkpoints taken every 8 tokens; arithmetic fp32.
 * Deterministic: the same inputs give bit-identical gradients.
 *
 *   q, k, v, log_alpha, beta, initial_state, cu_seqlens, total_T, N, H: as for
 *              kda_chunk_fwd (dk == dv == 128 only: KDA_ERR_UNSUPPORTED otherwise).
 *   d_out      device [total_T, H, dv], dtype qkv_dtype: gradient of the outputs.
 *   d_final_state  device fp32 [N, H, dk, dv] or NULL (zero).
 *   dq, dk, dv, d_log_alpha   device fp32 [total_T, H, 128], written.
 *   d_beta     device fp32 [total_T, H], written.
 *   d_initial_state  device fp32 [N, H, dk, dv] or NULL (not written): gradient of the
 *              state before each sequence (d_final_state for an empty sequence).
 *   workspace  device, >= kda_chunk_bwd_workspace(...) bytes, 16-byte aligned.
 * Outputs must not overlap the inputs. Pointers 16-byte aligned (beta, d_beta: 4).
 * Returns KDA_OK once the work is enqueued; bad cu_seqlens set KDA_DEVFLAG_BAD_SEQLENS
 * in the workspace status word and leave the outputs unwritten.
 */
KDA_API kda_status kda_chunk_bwd(const void* q, const void* k, const void* v, kda_dtype qkv_dtype,
                                 const float* log_alpha, const float* beta, const float* initial_state,
                                 const int32_t* cu_seqlens, int64_t total_T, int N, int H, int dk, int dv,
                                 const void* d_out, const float* d_final_state, float* dq, float* dk_out,
                                 float* dv_out, float* d_log_alpha, float* d_beta, float* d_initial_state,
                                 void* workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * Reads the device status word kept in `workspace` (KDA_DEVFLAG_* bits) after
 * synchronising `stream`, and clears it. Returns KDA_ERR_RANGE when any bit
 * was set, KDA_OK otherwise; *flags (if not NULL) receives the bits.
 */
KDA_API kda_status kda_workspace_status(void* workspace, kda_stream_t stream, uint32_t* flags);

/*
 * Diagnostic of the library's failure path (the pages have no counterpart). Every
 * wait inside the kernels (on an mbarrier: a tensor-core commit, a bulk copy, a
 * hand-over between warp groups) is bounded: after its budget it sets
 * KDA_DEVFLAG_WAIT_TIMEOUT in the call's status word and the kernel returns, so a
 * lost arrival ends as a status the host can read rather than as a hung GPU. This
 * call launches one thread that waits, with that same bounded wait and a budget of
 * budget_us microseconds, on an mbarrier that nothing arrives at: it always runs
 * out, sets the bit in `workspace`'s status word (cleared first) and returns.
 *   workspace  device, >= 256 bytes, 16-byte aligned (any workspace of this library)
 *   budget_us  1 .. 2,000,000
 * Read the result with kda_workspace_status (KDA_ERR_RANGE, flags =
 * KDA_DEVFLAG_WAIT_TIMEOUT).
 */
KDA_API kda_status kda_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint32_t budget_us,
                                             kda_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
