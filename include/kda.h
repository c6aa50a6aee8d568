/*
 * kda.h -- C ABI of libkda, a B200 (sm_100a) library for the Kimi Delta
 * Attention (KDA) gated delta-rule recurrence.
 *
 * The operation (sources: the K3 article summaries on the xhh.club tag page,
 * items "KDA recurrence form", "chunkwise parallel algorithm" and "3:1
 * hybrid"; section 6 of the nlpx.cn K3 paper walkthrough).  Each head keeps a
 * dk x dv fp32 state S (row = key channel).  For every token t of a sequence:
 *
 *     l_t = max(log_alpha_t, -5)                     per key channel
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp(l_t)) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t
 *
 * optionally followed by the per-head RMSNorm and full-rank sigmoid gate
 *     y_t = o_t / sqrt(mean_j o_tj^2 + eps) * w * sigmoid(g_t).
 * Prefill runs the chunkwise form (64-token chunks: matrix products inside a
 * chunk, a recurrence between chunks); decode runs the recurrent form.
 *
 * Conventions for every entry point:
 *  - Pointers are DEVICE pointers owned by the caller, unless stated.  The
 *    library never allocates, frees or keeps them past the call.
 *  - Element layout is token-major, head-minor: [B, T, H, d] (contiguous).
 *    beta is [B, T, H].  States are fp32 [N, H, dk, dv], row = key channel.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call is asynchronous on that stream and never
 *    synchronises, except kda_query_status.
 *  - Arguments are checked on the host before any launch; a rejected call
 *    launches nothing and returns a negative kda_status.  A failed launch
 *    returns KDA_ERR_CUDA (cudaGetLastError is cleared into the return code).
 *    Errors detected on the device (a bounded wait that expired, cu_seqlens
 *    that contradict T or max_seqlen) are recorded in a status word inside
 *    the workspace and read back with kda_query_status.
 *  - Supported shapes: dk = dv = 128.  Supported dtypes: inputs KDA_F32 or
 *    KDA_BF16 (all of q, k, v, log_alpha, beta, gate share in_dtype);
 *    outputs KDA_F32 or KDA_BF16.  Every pointer must be 16-byte aligned.
 *  - Outputs must not alias inputs, except where stated (in-place states).
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

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = -1, /* null pointer, bad size, bad dtype */
    KDA_ERR_UNSUPPORTED = -2, /* shape outside what the kernels implement */
    KDA_ERR_MISALIGNED = -3,  /* a pointer is not 16-byte aligned */
    KDA_ERR_WORKSPACE = -4,   /* workspace missing or smaller than required */
    KDA_ERR_CUDA = -5,        /* a CUDA runtime call or launch failed */
    KDA_ERR_TIMEOUT = -6,     /* device: a bounded wait gave up */
    KDA_ERR_DEVICE_ARG = -7   /* device: cu_seqlens inconsistent with T / max_seqlen */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/* Human-readable name of a kda_status value (static string, never NULL). */
KDA_API const char* kda_status_string(int status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
KDA_API int kda_version(void);

/*
 * kda_chunk_fwd_workspace_size -- bytes of device workspace kda_chunk_fwd needs.
 *
 *   T, H, dk, dv   as for kda_chunk_fwd (T = tokens per sequence for fixed
 *                  length, total packed tokens for varlen)
 *   n_seqs         number of sequences N (B for fixed length)
 *   max_seqlen     longest sequence (T for fixed length)
 *   bytes_min      out: the smallest workspace accepted (one 64-token chunk
 *                  of every sequence per pass)
 *   bytes_full     out: the workspace that lets one pass cover every chunk
 *                  of every sequence (fewest launches)
 * Any size in [bytes_min, inf) works; larger workspaces need fewer passes.
 */
KDA_API kda_status kda_chunk_fwd_workspace_size(int64_t T, int H, int dk, int dv, int n_seqs,
                                        int64_t max_seqlen, size_t* bytes_min,
                                        size_t* bytes_full);

/*
 * kda_chunk_fwd -- chunkwise prefill / training forward of the KDA recurrence.
 * Defined by the "chunkwise parallel algorithm" item of the K3 article
 * summaries (xhh.club tag page): 64-token chunks, state recurrence between
 * chunks, matrix products inside a chunk, per-step log-decay bounded below by
 * -5, 16-token diagonal tiles in BF16 matrix multiplies.
 *
 *   q, k, log_alpha  [B, T, H, dk]   in_dtype
 *   v                [B, T, H, dv]   in_dtype
 *   beta             [B, T, H]       in_dtype, values in [0, 1]
 *   init_state       [N, H, dk, dv]  fp32, NULL = zero state
 *   o                [B, T, H, dv]   out_dtype: o, or y when gate != NULL
 *   final_state      [N, H, dk, dv]  fp32, NULL = not returned.  May alias
 *                                    init_state (updated in place).
 *   B, T             batch and tokens per sequence; for varlen B = 1 and T
 *                    = total packed tokens
 *   H, dk, dv        heads and head dims (dk = dv = 128)
 *   cu_seqlens       device int32 [n_seqs + 1] (cu[0] = 0, non-decreasing,
 *                    cu[n_seqs] = T), or NULL for B fixed-length sequences
 *   n_seqs           number of sequences when cu_seqlens != NULL (else B)
 *   max_seqlen       host upper bound on any sequence length (T when
 *                    cu_seqlens == NULL); lengths above it are a device error
 *   scale            output scale (1.0 for the plain recurrence)
 *   gate             [B, T, H, dv] in_dtype, or NULL: when given, the per-head
 *                    RMSNorm (over dv) and sigmoid gate are applied and y is
 *                    written to o
 *   norm_weight      [dv] fp32 RMSNorm weight shared by heads, NULL = ones
 *   eps              RMSNorm epsilon
 *   workspace        device buffer of workspace_bytes >=
 *                    kda_chunk_fwd_workspace_size(...).bytes_min, 256-byte
 *                    aligned.  Holds the per-chunk intermediates and the
 *                    device status word; its contents on entry are ignored.
 *   stream           cudaStream_t as void*
 * Zero-length sequences are allowed (final state = initial state).
 */
KDA_API kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const void* log_alpha,
                         const void* beta, const float* init_state, void* o,
                         float* final_state, int B, int64_t T, int H, int dk, int dv,
                         const int32_t* cu_seqlens, int n_seqs, int64_t max_seqlen,
                         kda_dtype in_dtype, kda_dtype out_dtype, float scale,
                         const void* gate, const float* norm_weight, float eps,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * kda_chunk_fwd_ckpt -- kda_chunk_fwd that also emits state checkpoints for a
 * prefix cache (the "training and inference systems" item of the K3 article
 * summaries: states cached at 512-token boundaries).  Arguments as
 * kda_chunk_fwd, plus:
 *
 *   checkpoints  NULL (then identical to kda_chunk_fwd), or fp32
 *                [n_seqs, n_ckpt, H, dk, dv] with n_ckpt = max_seqlen /
 *                ckpt_tokens (fixed length: T / ckpt_tokens), 16-byte aligned.
 *                Checkpoint j of sequence n is the state after that sequence's
 *                first (j + 1) * ckpt_tokens tokens (initial state included);
 *                checkpoints beyond a sequence's length are not written.
 *   ckpt_tokens  checkpoint spacing in tokens, a positive multiple of 64
 *                (the chunk length); KDA_ERR_INVALID_ARG otherwise.
 */
KDA_API kda_status kda_chunk_fwd_ckpt(const void* q, const void* k, const void* v, const void* log_alpha,
                              const void* beta, const float* init_state, void* o,
                              float* final_state, int B, int64_t T, int H, int dk, int dv,
                              const int32_t* cu_seqlens, int n_seqs, int64_t max_seqlen,
                              kda_dtype in_dtype, kda_dtype out_dtype, float scale,
                              const void* gate, const float* norm_weight, float eps,
                              float* checkpoints, int64_t ckpt_tokens,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * kda_chunk_fwd_segmented -- kda_chunk_fwd with every sequence cut into
 * `segments` segments of whole chunks that are walked in parallel: the
 * segment-parallel (associative scan) form of the prefill ("training and
 * inference systems" item of the K3 article summaries: context parallelism as a
 * prefix scan of segment transitions; the nlpx.cn walkthrough, §6: KCP).
 * Pass 1 computes, per (sequence, segment, head), the segment's affine state
 * map S -> M S + B; pass 2 walks each segment from the initial state folded
 * through the maps of the segments before it.  Useful when n_seqs * H is small
 * next to the GPU (the plain walk has 4 * n_seqs * H independent chains).
 * Arguments as kda_chunk_fwd plus `segments` (>= 1; 1 is kda_chunk_fwd); the
 * workspace must hold kda_chunk_fwd_segmented_workspace_size bytes (every chunk
 * at once plus the segment maps).  Results equal kda_chunk_fwd's up to bf16
 * rounding of the segment maps.
 */
KDA_API kda_status kda_chunk_fwd_segmented(const void* q, const void* k, const void* v,
                                   const void* log_alpha, const void* beta,
                                   const float* init_state, void* o, float* final_state,
                                   int B, int64_t T, int H, int dk, int dv,
                                   const int32_t* cu_seqlens, int n_seqs, int64_t max_seqlen,
                                   kda_dtype in_dtype, kda_dtype out_dtype, float scale,
                                   const void* gate, const float* norm_weight, float eps,
                                   int segments, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * kda_chunk_fwd_segmented_workspace_size -- workspace bytes for
 * kda_chunk_fwd_segmented (arguments as kda_chunk_fwd_workspace_size plus
 * segments).
 */
KDA_API kda_status kda_chunk_fwd_segmented_workspace_size(int64_t T, int H, int dk, int dv, int n_seqs,
                                                  int64_t max_seqlen, int segments,
                                                  size_t* bytes);

/*
 * Context parallelism across devices (KCP: the nlpx.cn K3 walkthrough, §6; the
 * "training and inference systems" item of the K3 article summaries: context
 * parallelism as a prefix scan of segment transitions).  Every sequence is cut
 * into consecutive token segments, segment r on device r.  Segment r's effect
 * on the state is affine, S -> M_r S + B_r, so each device
 *   1. kda_kcp_transition: runs the chunk-local work over its segment, keeps it
 *      in the workspace and writes (M_r, B_r) in fp32;
 *   2. exchanges the maps (an all-gather in device order; the library does no
 *      communication);
 *   3. kda_kcp_compose: folds the maps of devices 0 .. r-1 over the sequences'
 *      initial state into its own initial state;
 *   4. kda_kcp_finish: walks its kept chunks from that state, with outputs.
 * Device r's outputs then equal those of kda_chunk_fwd over the whole
 * sequence (up to fp32 rounding of the composition and bf16 rounding of the
 * map's state image inside the walk), and the last device's final state is
 * the sequence's.  Arguments as kda_chunk_fwd, for this device's segment.
 *
 * kda_kcp_workspace_size -- bytes of the workspace that steps 1 and 4 share
 * (every chunk's slot at once: kda_chunk_fwd_workspace_size's bytes_full).
 */
KDA_API kda_status kda_kcp_workspace_size(int64_t T, int H, int dk, int dv, int n_seqs, int64_t max_seqlen,
                                          size_t* bytes);

/*
 * kda_kcp_transition -- step 1.  Inputs as kda_chunk_fwd (q and scale are used:
 * the kept chunk work includes the output terms).
 *
 *   transition  [2, N, H, dk, dk] fp32, device, caller-owned: [0] = M (dk x dk),
 *               [1] = B (dk x dv) with S_out = M S_in + B per (sequence, head);
 *               an empty segment gives M = I, B = 0
 *   workspace   >= kda_kcp_workspace_size bytes, 256-byte aligned; it holds the
 *               chunk slots until kda_kcp_finish has run on the same stream
 *
 * Errors as kda_chunk_fwd (device-side ones land in the workspace status word).
 */
KDA_API kda_status kda_kcp_transition(const void* q, const void* k, const void* v, const void* log_alpha,
                                      const void* beta, int B, int64_t T, int H, int dk, int dv,
                                      const int32_t* cu_seqlens, int n_seqs, int64_t max_seqlen,
                                      kda_dtype in_dtype, float scale, float* transition, void* workspace,
                                      size_t workspace_bytes, void* stream);

/*
 * kda_kcp_compose -- step 3:  S = init_state (zero when NULL), then for
 * j = 0 .. n_prev-1:  S = M_j S + B_j;  state_in = S.
 *
 *   transitions [R, 2, N, H, dk, dk] fp32, device: the gathered maps in device
 *               order (R >= n_prev; may be NULL when n_prev == 0)
 *   init_state  [N, H, dk, dv] fp32 or NULL; state_in [N, H, dk, dv] fp32 (output)
 *
 * KDA_ERR_INVALID_ARG for n_prev < 0 or missing buffers, KDA_ERR_MISALIGNED
 * for pointers not 16-byte aligned.
 */
KDA_API kda_status kda_kcp_compose(const float* transitions, int n_prev, const float* init_state,
                                   float* state_in, int n_seqs, int H, int dk, int dv, void* stream);

/*
 * kda_kcp_finish -- step 4: the walk of kda_chunk_fwd over the chunk slots
 * that kda_kcp_transition left in `workspace` (same B, T, H, cu_seqlens,
 * n_seqs, max_seqlen and workspace), starting from state_in (NULL = zero).
 * o, final_state, gate, norm_weight, eps and the dtypes as kda_chunk_fwd;
 * in_dtype is the gate's dtype.  The workspace status word carries step 1's
 * device-side errors too.
 */
KDA_API kda_status kda_kcp_finish(const float* state_in, void* o, float* final_state, int B, int64_t T, int H,
                                  int dk, int dv, const int32_t* cu_seqlens, int n_seqs, int64_t max_seqlen,
                                  kda_dtype in_dtype, kda_dtype out_dtype, const void* gate,
                                  const float* norm_weight, float eps, void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * kda_chunk_bwd -- gradients of kda_chunk_fwd (without the gate) with respect
 * to q, k, v, log_alpha, beta and the initial state, given dL/do and dL/d(final
 * state).  The pages give no backward pass; this is the exact gradient of the
 * forward definition, computed chunkwise: the forward walk is recomputed (chunk
 * slots and chunk-boundary states kept in the workspace), a reverse walk forms
 * dL/d(state) at every chunk end, and a chunk-local kernel forms the token
 * gradients.  The clamp l = max(log_alpha, -5) passes the gradient where
 * log_alpha >= -5 and blocks it below.
 *
 *   q, k, v, log_alpha, beta, init_state, B, T, H, cu_seqlens, n_seqs,
 *   max_seqlen, in_dtype, scale   as kda_chunk_fwd
 *   d_o           [B, T, H, dv] in_dtype: dL/do (device)
 *   d_final_state [N, H, dk, dv] fp32 or NULL (zero)
 *   dq, dk, dlog_alpha [B, T, H, dk] fp32; dv [B, T, H, dv] fp32; dbeta [B, T, H]
 *                 fp32 (outputs, caller-owned device memory)
 *   d_init_state  [N, H, dk, dv] fp32 or NULL: dL/d(initial state)
 *   workspace     >= kda_chunk_bwd_workspace_size bytes, 256-byte aligned
 *
 * Errors as kda_chunk_fwd; device-side ones land in the workspace status word.
 */
KDA_API kda_status kda_chunk_bwd(const void* q, const void* k, const void* v, const void* log_alpha,
                                 const void* beta, const float* init_state, const void* d_o,
                                 const float* d_final_state, float* dq, float* dk, float* dv,
                                 float* dlog_alpha, float* dbeta, float* d_init_state, int B, int64_t T,
                                 int H, int dk_dim, int dv_dim, const int32_t* cu_seqlens, int n_seqs,
                                 int64_t max_seqlen, kda_dtype in_dtype, float scale, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * kda_chunk_bwd_workspace_size -- workspace bytes of kda_chunk_bwd: the
 * forward's whole-sequence workspace plus, per chunk and head, the state at the
 * chunk's start and the state gradient at its end, each kept as a bf16 128 x 128
 * operand image (arguments as kda_chunk_fwd_workspace_size).
 */
KDA_API kda_status kda_chunk_bwd_workspace_size(int64_t T, int H, int dk, int dv, int n_seqs, int64_t max_seqlen,
                                                size_t* bytes);

/*
 * kda_decode_step -- one recurrent step for Bd independent sequences
 * ("decode uses the recurrent form", chunkwise-algorithm item of the K3
 * article summaries).  The state is read once and written once, in place.
 *
 *   state        [Bd, H, dk, dv] fp32, updated in place
 *   q, k, log_alpha [Bd, H, dk]; v [Bd, H, dv]; beta [Bd, H]   in_dtype
 *   o            [Bd, H, dv] out_dtype (y when gate != NULL)
 *   gate         [Bd, H, dv] in_dtype or NULL; norm_weight [dv] fp32 or NULL
 */
KDA_API kda_status kda_decode_step(float* state, const void* q, const void* k, const void* v,
                           const void* log_alpha, const void* beta, void* o, int Bd, int H,
                           int dk, int dv, kda_dtype in_dtype, kda_dtype out_dtype,
                           float scale, const void* gate, const float* norm_weight,
                           float eps, void* stream);

/*
 * kda_decode_steps -- n_steps consecutive recurrent steps for Bd independent
 * sequences in one call: verification of n_steps draft tokens in speculative
 * decoding, or plain decode of several tokens.  (Decode runs the recurrent
 * form, chunkwise-algorithm item of the K3 article summaries; speculative
 * decoding with state rollback is the "training and inference systems" item.)
 * Each (sequence, head) state is read once and written once for all steps.
 *
 *   state        [Bd, H, dk, dv] fp32: the state before step 0; on return the
 *                state after the last step
 *   q, k, log_alpha, gate [n_steps, Bd, H, dk]; v [n_steps, Bd, H, dv];
 *   beta [n_steps, Bd, H]          in_dtype (step-major)
 *   o            [n_steps, Bd, H, dv] out_dtype (y when gate != NULL)
 *   step_states  NULL, or [n_steps, Bd, H, dk, dv] fp32: the state after each
 *                step (step_states[n_steps - 1] equals the final state).  To
 *                roll back to "accepted the first a tokens" (1 <= a <= n_steps)
 *                copy step_states[a - 1] into the state; keep a copy of the
 *                incoming state to reject every draft token.
 * Errors as kda_decode_step; n_steps == 0 or Bd == 0 does nothing.
 */
KDA_API kda_status kda_decode_steps(float* state, const void* q, const void* k, const void* v,
                            const void* log_alpha, const void* beta, void* o, int n_steps,
                            int Bd, int H, int dk, int dv, kda_dtype in_dtype,
                            kda_dtype out_dtype, float scale, const void* gate,
                            const float* norm_weight, float eps, float* step_states,
                            void* stream);

/*
 * kda_gate_norm -- per-head RMSNorm over dv followed by the full-rank sigmoid
 * output gate ("KDA recurrence form" and "3:1 hybrid" items of the K3
 * article summaries):  y = o / sqrt(mean(o^2) + eps) * w * sigmoid(g).
 *
 *   o      [rows, dv] in_dtype (rows = B*T*H)
 *   gate   [rows, dv] in_dtype
 *   norm_weight [dv] fp32 or NULL (ones)
 *   y      [rows, dv] out_dtype; may alias o exactly (in place)
 */
KDA_API kda_status kda_gate_norm(const void* o, const void* gate, const float* norm_weight, float eps,
                         void* y, int64_t rows, int dv, kda_dtype in_dtype,
                         kda_dtype out_dtype, void* stream);

/*
 * kda_query_status -- synchronises `stream`, reads the device status word of
 * a kda_chunk_fwd workspace, clears it and returns it (KDA_OK when no device
 * error was recorded).  This is the only call that blocks the host.
 */
KDA_API kda_status kda_query_status(void* workspace, void* stream);

/*
 * kda_test_drop_tile_load -- test hook for the device-side failure path (no
 * counterpart on the pages).  The next kda_chunk_fwd-family call with bf16
 * inputs in this process runs its chunk-local kernel with one change: CTA 0
 * does not issue one of the four tile loads of its first item, and its wait
 * for them gives up after wait_limit_ns (1e3 .. 1e9 ns) instead of the usual
 * second.  That CTA then stops; the call returns KDA_OK, its outputs are
 * undefined, and kda_query_status on its workspace returns KDA_ERR_TIMEOUT.
 * The process and the GPU context stay usable: the next call is normal.
 * wait_limit_ns = 0 cancels a pending drop.  Host-side only; not
 * thread-safe.  KDA_ERR_INVALID_ARG for any other limit outside the range.
 */
KDA_API kda_status kda_test_drop_tile_load(unsigned long long wait_limit_ns);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that cannot allocate
 * device memory.  (No counterpart on the pages: it is a packaging of
 * kda_chunk_fwd, not part of the method.)
 *
 * Who needs it: hosts that hand a plugin its inputs and outputs but no way to
 * get device scratch -- e.g. a framework whose memory pool already owns all
 * free device memory, or a runtime that forbids cudaMalloc on its hot path
 * because cudaMalloc can synchronise the device.  Here the scratch is a
 * static array of KDA_NOALLOC_SCRATCH_BYTES inside libkda's own device
 * memory, so there is no workspace argument and the call allocates nothing.
 *
 * Arguments, layouts and results are exactly those of kda_chunk_fwd minus
 * (workspace, workspace_bytes).  The caller still owns every input and output.
 *  - Limit: the problem must fit the static scratch, i.e.
 *    kda_chunk_fwd_workspace_size(...).bytes_min <= KDA_NOALLOC_SCRATCH_BYTES
 *    (roughly n_seqs * H <= 400).  Larger problems
 *    return KDA_ERR_WORKSPACE before any CUDA call; larger scratch than the
 *    minimum only means fewer passes.
 *  - The array is reserved on each GPU that loads this part of the library and
 *    is held until the process exits.  The first call on a device looks up the
 *    array's device address (cudaGetSymbolAddress) with that device current;
 *    make that first call before any stream capture on that device.
 *  - Every call on a device shares the one array, which keeps the previous
 *    call's contents (the call clears the parts that must start at zero
 *    itself).  Calls that overlap on the GPU (different streams without
 *    ordering, or different host threads) race on it: order them.
 *  - Errors the kernels detect on the device (a bounded wait that gave up,
 *    cu_seqlens that contradict T or max_seqlen) are recorded in a status word
 *    at the start of the static array; read them with
 *    kda_chunk_fwd_noalloc_query_status (kda_query_status takes a workspace,
 *    and this entry point has none).  Each call clears the word first, so it
 *    describes the last call on the device.
 *  - The array's device address is cached per device; after a cudaDeviceReset
 *    the module is unloaded and the cached address is stale, so do not call
 *    this entry point again in that process after a reset.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

KDA_API kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                 const void* log_alpha, const void* beta,
                                 const float* init_state, void* o, float* final_state,
                                 int B, int64_t T, int H, int dk, int dv,
                                 const int32_t* cu_seqlens, int n_seqs, int64_t max_seqlen,
                                 kda_dtype in_dtype, kda_dtype out_dtype, float scale,
                                 const void* gate, const float* norm_weight, float eps,
                                 void* stream);

/*
 * kda_chunk_fwd_noalloc_query_status -- synchronises `stream` and returns the
 * device status word of the last kda_chunk_fwd_noalloc call on the current
 * device (then clears it): KDA_OK, KDA_ERR_TIMEOUT or KDA_ERR_DEVICE_ARG, as
 * kda_query_status does for a workspace.  Allocates nothing.  Returns
 * KDA_ERR_CUDA if the array's address cannot be looked up.
 */
KDA_API kda_status kda_chunk_fwd_noalloc_query_status(void* stream);

/*
 * Per-kernel device timing (a measurement aid, off by default).
 * kda_profile_enable(1) makes every later launch of this library bracket each
 * of its kernels with CUDA events on the launch stream.  kda_profile_read
 * synchronises on those events, writes one entry per kernel kind that ran
 * (name, number of launches, summed device milliseconds) into out[0 ..
 * max_entries), stores the count in *n_entries and resets the counters.
 * Host-side only; not thread-safe.
 */
typedef struct {
    char name[16];
    int launches;
    double ms;
} kda_kernel_time;

KDA_API kda_status kda_profile_enable(int on);
KDA_API kda_status kda_profile_read(kda_kernel_time* out, int max_entries, int* n_entries);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
