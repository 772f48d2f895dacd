/*
 * kda.h -- C ABI of libkda, the B200 (sm_100a) Kimi Delta Attention forward.
 *
 * KDA is a per-head recurrence over a matrix state S in R^{dk x dv}:
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t = scale * S_t^T q_t,              alpha_t = exp(g_t) per key channel
 *
 * The update is the "combined form" of section 3.3 of "Kimi Linear's Hybrid
 * Linear Attention Architecture: A Technical Breakdown" (decay first, then the
 * erase along k_t and the write), with the state oriented dk x dv as in the
 * update printed in "Kimi Linear: How Moonshot AI Built a Hybrid Attention
 * Architecture That Beats Full Attention" (beta_t k_t v_t^T).  The query reads
 * the state after its own token's write ("Kimi Linear" explainer,
 * math.kryvik.com, "Step 4: Query").  Prefill evaluates the recurrence in the
 * chunkwise form of section 4 of the Baidu breakdown (state passing across
 * chunks, causal intra-chunk output); decode is one step of the recurrence.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All pointers are DEVICE pointers (cudaMalloc / torch CUDA tensors) on the
 *   current device, row-major and contiguous, 16-byte aligned (beta: 4-byte);
 *   kda_chunk_fwd_host alone takes host pointers.
 * - bf16 tensors are passed as void* holding IEEE bfloat16 (uint16 bits).
 * - The caller owns every buffer it passes.  The library keeps no pointer to
 *   them after a call returns.  Library-owned device memory: one 4-byte status
 *   word per device (part of the module image), and the prefill workspace
 *   described at kda_chunk_fwd_workspace_bytes().
 * - Work is enqueued on `stream` (a cudaStream_t, NULL = legacy default
 *   stream) and the call returns without synchronising.  The return value
 *   reports argument validation and launch errors only.  Device-side
 *   conditions (a bounded wait that gave up) are reported by
 *   kda_stream_status().
 * - Supported sizes: dk, dv in {64, 128}; B, H >= 1; T >= 0.  Anything else
 *   returns KDA_ERR_UNSUPPORTED (or KDA_ERR_INVALID_ARG for negative sizes
 *   and NULL required pointers) without enqueueing work.
 * - Value domain: g <= 0 and finite, beta in [0, 1].  Keys are used as given
 *   (the caller L2-normalises them if the model does).  Results are exact up
 *   to rounding for every such g.  A 64-token chunk in which some key channel
 *   loses more than 80 of log-decay over 8 consecutive tokens (in an aligned
 *   16-token block: tokens 1..8 or 9..15 of it) takes a slower exact path for
 *   its intra-chunk terms (about one such chunk in a million at the decays of
 *   trained models; none in the workloads here).
 * - Operand range of the prefill.  Three intermediate operands of the tensor
 *   contractions are fp16 (10-bit mantissa, largest finite value 65504): the
 *   causal block P (entries bounded by |q_i| |k_j|), the decayed keys
 *   k * e^{Gamma_C - Gamma} (bounded by |k|), and the corrected values
 *   v_new = beta (v - (decayed S)^T k)-combinations, bounded by about
 *   max|v| + |k| max|S column|.  So the prefill needs |q|, |k| <= ~1 (unit
 *   keys and queries, as the model uses) and |v| and the state's entries well
 *   below 6.5e4; within that, its relative error does not depend on the scale
 *   of v and h0 (the method is linear in them).  Decode has no such limit.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>

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
    KDA_ERR_INVALID_ARG = 1, /* NULL required pointer, negative size           */
    KDA_ERR_UNSUPPORTED = 2, /* dk/dv outside {64,128}, other unsupported shape */
    KDA_ERR_ALIGNMENT = 3,   /* a pointer below its required alignment        */
    KDA_ERR_CUDA = 4,        /* a CUDA runtime/driver call or launch failed    */
    KDA_ERR_TIMEOUT = 5,     /* a device-side bounded wait gave up             */
    KDA_ERR_SCRATCH_LIMIT = 6, /* kda_chunk_fwd_noalloc: problem exceeds its fixed scratch */
    KDA_ERR_BOUNDS = 7       /* debug build (libkda_debug.so): an index check failed */
} kda_status;

/*
 * kda_chunk_fwd -- chunkwise prefill over whole sequences.
 *
 *   q, k  : bf16 [B, T, H, dk]
 *   v     : bf16 [B, T, H, dv]
 *   g     : fp32 [B, T, H, dk]   log-decay, g = log(alpha) <= 0
 *   beta  : fp32 [B, T, H]       write/erase strength in [0, 1]
 *   scale : readout scale (commonly dk^-0.5)
 *   h0    : fp32 [B, H, dk, dv]  initial state, or NULL for a zero state
 *   out   : bf16 [B, T, H, dv]   o_t for every token (written)
 *   hT    : fp32 [B, H, dk, dv]  final state, or NULL to skip; may alias h0
 *           (h0 is read in full before hT is written, per (b, h))
 *   stream: cudaStream_t
 *
 * Internally each sequence is cut into chunks of 64 tokens; the last chunk of
 * a sequence may be partial.  Per segment of chunks, one kernel builds every
 * chunk's state-independent pieces in parallel (decay-scaled operands, the
 * intra-chunk blocks, the inverse of the unit-lower system and the WY
 * factors) into the workspace; another walks the chunks of each (b, h) in
 * order, carrying the state in fp32.  With few (b, h) and enough chunks the
 * walk is two-level: the segment is cut into parts, every part's transition
 * (dk x dk) and zero-start state are formed in parallel, a short sequential
 * fix-up gives each part its start state, and the parts then produce their
 * outputs in parallel (the "chunked parallel" scheme of the "Kimi Linear"
 * explainer, math.kryvik.com).  The chunk contractions run on the tcgen05
 * tensor cores with fp32 accumulation.  T == 0 copies h0 to hT
 * (or zeroes hT) and writes no output; q, k, v, g, beta and out are then not
 * read and may be NULL.
 *
 * Workspace: the first call on a device, and any call that needs more than
 * the workspace held so far, allocates it with cudaMalloc (freeing the old
 * one first, which synchronises the device), so make such a call before any
 * stream capture.  Calls on different streams are ordered on the workspace by
 * an event.  Allocation failure returns KDA_ERR_CUDA.
 */
KDA_API int kda_chunk_fwd(const void *q, const void *k, const void *v,
                  const float *g, const float *beta, float scale,
                  const float *h0, void *out, float *hT,
                  int B, int T, int H, int dk, int dv, void *stream);

/*
 * kda_decode_step -- one recurrent step for every (b, h), state updated in place.
 *
 *   q, k  : bf16 [B, H, dk]
 *   v     : bf16 [B, H, dv]
 *   g     : fp32 [B, H, dk]
 *   beta  : fp32 [B, H]
 *   scale : readout scale
 *   state : fp32 [B, H, dk, dv]  S_{t-1} on entry, S_t on return
 *   out   : bf16 [B, H, dv]      o_t
 *   stream: cudaStream_t
 *
 * The state layout is the one kda_chunk_fwd uses for h0/hT, so a decode can
 * continue a prefill directly.  This is the recurrence itself, evaluated in
 * fp32: decay each key row of S, project on k, erase-and-write, read with q.
 */
KDA_API int kda_decode_step(const void *q, const void *k, const void *v,
                    const float *g, const float *beta, float scale,
                    float *state, void *out,
                    int B, int H, int dk, int dv, void *stream);

/*
 * kda_gdn_chunk_fwd, kda_gdn_decode_step -- the scalar-gate form (Gated
 * DeltaNet): one log-decay per token and head, shared by every key channel,
 * i.e. alpha_t = exp(g_t) * 1 in the recurrence above.
 *
 *   g : fp32 [B, T, H] (prefill) or [B, H] (decode), 4-byte aligned
 *
 * Every other argument, layout, result and error code is that of kda_chunk_fwd
 * and kda_decode_step respectively (the prefill shares their workspace); the
 * results are those of the per-channel entry points given g broadcast over dk.
 * The state-independent prep reads 4 bytes of gate per token and head instead
 * of 4 dk.
 */
KDA_API int kda_gdn_chunk_fwd(const void *q, const void *k, const void *v,
                  const float *g, const float *beta, float scale,
                  const float *h0, void *out, float *hT,
                  int B, int T, int H, int dk, int dv, void *stream);
KDA_API int kda_gdn_decode_step(const void *q, const void *k, const void *v,
                    const float *g, const float *beta, float scale,
                    float *state, void *out,
                    int B, int H, int dk, int dv, void *stream);

/*
 * kda_chunk_fwd_raw, kda_decode_step_raw -- the prefill and the decode step
 * with the gate prologue fused: they take the raw projections a KDA layer
 * produces and form the recurrence's inputs themselves, per token and head:
 *
 *   g     = -gate_c * softplus(g_raw)      per key channel (so g <= 0)
 *   beta  = sigmoid(beta_raw)
 *   q, k  = q_raw / |q_raw|, k_raw / |k_raw|  (L2 over dk, norms floored at
 *           1e-12; the normalised values are rounded to bf16 as stored inputs)
 *
 * gate_c = 1 gives alpha = e^g = sigmoid(-g_raw): the channel-wise sigmoid gate
 * of the "Kimi Linear" explainer (math.kryvik.com), "Step 2: Per-Channel
 * Decay", with the sign folded into the projection; the decay is the
 * fine-grained gate of section 3.2 of "Kimi Linear's Hybrid Linear Attention
 * Architecture: A Technical Breakdown".  The kernels apply it where they load
 * g, beta, q and k, so the unfused values never go through memory.
 *
 *   q, k, v, g_raw, beta_raw: the layouts and dtypes of kda_chunk_fwd
 *           (prefill) and kda_decode_step (decode); q and k need not be
 *           normalised, g_raw and beta_raw are any finite fp32 values
 *   gate_c: >= 0 and finite, else KDA_ERR_INVALID_ARG
 *
 * Everything else (arguments, workspace, errors, value range) is that of
 * kda_chunk_fwd and kda_decode_step; the results are theirs given the
 * prologue's values.  Per key channel gates only.
 */
KDA_API int kda_chunk_fwd_raw(const void *q, const void *k, const void *v,
                  const float *g_raw, const float *beta_raw, float gate_c, float scale,
                  const float *h0, void *out, float *hT,
                  int B, int T, int H, int dk, int dv, void *stream);
KDA_API int kda_decode_step_raw(const void *q, const void *k, const void *v,
                  const float *g_raw, const float *beta_raw, float gate_c, float scale,
                  float *state, void *out,
                  int B, int H, int dk, int dv, void *stream);

/*
 * kda_chunk_bwd -- the backward pass of kda_chunk_fwd: the gradients of a
 * loss L with respect to q, k, v, g, beta and h0, given dL/dout and dL/dhT.
 * The pages describe training ("Kimi Linear" explainer, "Chunked
 * Processing": training speed comparable to FlashAttention) but print no
 * backward; this is reverse-mode differentiation of the recurrence of section
 * 3.3 of the Baidu breakdown, evaluated in its recurrent form: a forward walk
 * that stores the state every 8 tokens, then a backward walk over the tokens
 * that recomputes each token's state from checkpoints (two levels: a state
 * every 64 tokens from the forward walk, then per 64-token chunk a state every
 * 4 tokens).  fp32 arithmetic on CUDA cores, one CTA per (b, h).
 *
 *   q, k, v, g, beta, scale, h0 : the forward's inputs (layouts of kda_chunk_fwd)
 *   dout  : bf16 [B, T, H, dv]   dL/dout, or NULL (zero)
 *   dhT   : fp32 [B, H, dk, dv]  dL/dhT, or NULL (zero)
 *   dq, dk: bf16 [B, T, H, dk]   (written)
 *   dv    : bf16 [B, T, H, dv]
 *   dg    : fp32 [B, T, H, dk]   gradient of the log-decay
 *   dbeta : fp32 [B, T, H]
 *   dh0   : fp32 [B, H, dk, dv]  or NULL (not written)
 *
 * Workspace: the state checkpoints, B H (ceil(T / 64) + 16) dk dv fp32, and
 * each token's p = (Diag(alpha) S)^T k from the first pass, B H T dv fp32
 * (kda_chunk_bwd_workspace_bytes: 1.9 GB for B8 H32 T4096 d128, 51 GB for
 * B1 H32 T1M), held like the prefill's workspace (grown with cudaMalloc,
 * freed by kda_release_workspace).  T == 0 sets dh0 = dhT.
 * Errors as kda_chunk_fwd.
 */
KDA_API int kda_chunk_bwd(const void *q, const void *k, const void *v,
                  const float *g, const float *beta, float scale, const float *h0,
                  const void *dout, const float *dhT,
                  void *dq, void *dk, void *dv, float *dg, float *dbeta, float *dh0,
                  int B, int T, int H, int dk_, int dv_, void *stream);
KDA_API size_t kda_chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv);

/*
 * kda_chunk_fwd_varlen -- chunkwise prefill over a packed batch of N sequences
 * of different lengths, each with its own initial and final state.  This is
 * the serving form of the prefill: a batch of requests concatenated along the
 * token axis, each continuing from its cached recurrent state (the state cache
 * that takes the place of a KV cache in serving, paragraph on vLLM and LMCache
 * in "Kimi Linear: How Moonshot AI Built a Hybrid Attention Architecture That
 * Beats Full Attention").  Per sequence the result is exactly kda_chunk_fwd's.
 *
 *   q, k       : bf16 [T_total, H, dk]   the sequences back to back
 *   v          : bf16 [T_total, H, dv]
 *   g          : fp32 [T_total, H, dk]
 *   beta       : fp32 [T_total, H]
 *   cu_seqlens : int32 [N + 1], DEVICE memory, 4-byte aligned: sequence n
 *                holds tokens cu_seqlens[n] .. cu_seqlens[n+1] - 1; must
 *                start at 0, never decrease and end at T_total.  Empty
 *                sequences are allowed (their hT is their h0).
 *   h0         : fp32 [N, H, dk, dv] or NULL (zero states)
 *   out        : bf16 [T_total, H, dv]
 *   hT         : fp32 [N, H, dk, dv] or NULL; may alias h0
 *
 * Every sequence starts a new 64-token chunk, so chunks never mix sequences.
 * The library checks cu_seqlens on the device (the host never reads it):
 * offsets are clamped into a non-decreasing sequence within [0, T_total]
 * before any kernel uses them, so a bad array cannot make a kernel read or
 * write outside the buffers; the call then computes on the clamped offsets
 * and kda_stream_status() reports KDA_ERR_INVALID_ARG.  Uses the prefill
 * workspace (see kda_chunk_fwd_varlen_workspace_bytes); when the records of
 * all chunks do not fit in it, the chunks run in windows of kernel launches
 * and a state spanning windows is carried in hT (or in the workspace).
 * Other arguments, alignment rules and errors as kda_chunk_fwd (N < 1 or a
 * NULL cu_seqlens: KDA_ERR_INVALID_ARG).
 */
KDA_API int kda_chunk_fwd_varlen(const void *q, const void *k, const void *v,
                  const float *g, const float *beta, float scale,
                  const int *cu_seqlens, int N,
                  const float *h0, void *out, float *hT,
                  int T_total, int H, int dk, int dv, void *stream);

/*
 * kda_chunk_fwd_varlen_workspace_bytes -- device memory kda_chunk_fwd_varlen
 * holds for these sizes: counters, the steep-chunk list, the chunk geometry
 * (2 (N + 1) + T_total / 64 + N + 1 ints) and the records of one window of
 * chunks of every head (all chunks when they fit in 2 GiB), plus an fp32
 * state buffer [N, H, dk, dv] when there are several windows.  0 for
 * unsupported sizes or T_total == 0.
 */
KDA_API size_t kda_chunk_fwd_varlen_workspace_bytes(int N, int T_total, int H, int dk, int dv);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd without any device allocation.  The
 * method itself has no counterpart: this is a deployment variant for callers
 * that cannot allocate device memory at call time (a process whose device
 * memory is reserved up front by another allocator, or code that must not pay
 * the device-wide synchronisation of freeing a grown workspace).
 *
 * Same arguments, layouts, results and error codes as kda_chunk_fwd; the
 * outputs are bit-identical to it.  The chunk records live in a fixed 64 MiB
 * array per device that is part of the library's module image, so a long
 * sequence runs in several segments of a few kernel launches each.  Limit:
 * the records of one 64-token chunk of every (b, h) with their list entries
 * (B * H * 74,244 bytes), plus, when hT is NULL, the fp32 state [B, H, dk, dv]
 * carried between segments, must fit in 64 MiB (B * H <= 903 with hT given,
 * B * H <= 480 without, at dk = dv = 128); a larger problem returns
 * KDA_ERR_SCRATCH_LIMIT without enqueueing work.  The only parts of the
 * scratch that must start at zero, two counters, are cleared by each call.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it: make that first call before any stream
 * capture.  The scratch is shared by every call on the device, so calls that
 * overlap on the GPU (different streams, no ordering between them) race on
 * it and give wrong results; the caller orders them.
 */
KDA_API int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                  const float *g, const float *beta, float scale,
                  const float *h0, void *out, float *hT,
                  int B, int T, int H, int dk, int dv, void *stream);

/*
 * kda_chunk_fwd_host -- kda_chunk_fwd on HOST buffers: the one entry point
 * whose tensor pointers are host memory (q, k, v, g, beta, out as for
 * kda_chunk_fwd, h0 and hT fp32 [B, H, dk, dv] or NULL; any alignment).
 * Page-locked (pinned) buffers let the copies run asynchronously; pageable
 * ones work, with each copy staged synchronously by the runtime.
 *
 * The token axis runs in pieces of a multiple of 64 tokens (about 256 MB of
 * inputs each): the upload of a piece, the prefill of the one before it
 * (kda_chunk_fwd on device copies, continued from the previous piece's final
 * state: the recurrence of section 3.3 of the Baidu breakdown is exact across
 * any token boundary) and the download of the one before that overlap, on
 * two internal copy streams and `stream`.  Results equal those of
 * kda_chunk_fwd on the same inputs up to rounding at the piece boundaries
 * (identical chunks; the state passes through memory in fp32).
 *
 * Work is enqueued and the call returns: the host buffers must stay valid and
 * unchanged, and out / hT must not be read, until `stream` reaches the end of
 * this call's work (cudaStreamSynchronize or an event on it).  The library
 * holds device staging for two pieces and the state (grown on demand, freed
 * by kda_release_workspace) besides kda_chunk_fwd's own workspace; calls on a
 * device are ordered one after another.  T == 0 synchronises `stream` and sets
 * hT = h0 (or zero) on the host.  Return codes as kda_chunk_fwd.
 */
KDA_API int kda_chunk_fwd_host(const void *q, const void *k, const void *v,
                 const float *g, const float *beta, float scale,
                 const float *h0, void *out, float *hT,
                 int B, int T, int H, int dk, int dv, void *stream);

/*
 * kda_chunk_fwd_host_debug_piece -- test hook: pieces of `tokens` tokens for
 * kda_chunk_fwd_host (any positive count, not only multiples of 64); 0
 * restores the automatic size.  Process-wide.
 */
KDA_API void kda_chunk_fwd_host_debug_piece(int tokens);

/*
 * kda_chunk_fwd_workspace_bytes -- device memory kda_chunk_fwd holds for these
 * sizes: the per-chunk records (72.5 KB per 64-token chunk and (b, h)) of
 * the whole sequence when they fit in 2 GiB, else of two segments of as many
 * chunks as fit in 1 GiB each (at least one; the prep kernel of one segment
 * overlaps the state chain of the previous one on two internal streams),
 * plus then an fp32 state buffer [B, H, dk, dv], plus 256 bytes of counters.
 * 0 for unsupported sizes or T == 0.
 */
KDA_API size_t kda_chunk_fwd_workspace_bytes(int B, int T, int H, int dk, int dv);

/*
 * kda_release_workspace -- free the current device's prefill workspace and
 * kda_chunk_fwd_host's staging (the next call allocates them again).  cudaFree synchronises the device,
 * so no launched work still uses it.  KDA_OK, or KDA_ERR_CUDA.
 */
KDA_API int kda_release_workspace(void);

/* Human-readable name of a kda_status value (static string, never NULL). */
KDA_API const char *kda_status_string(int status);

/*
 * kda_stream_status -- synchronise `stream`, then read and clear the current
 * device's status word.  Returns KDA_OK, KDA_ERR_TIMEOUT when a kernel's
 * bounded wait gave up since the last call (that kernel's outputs are then
 * unspecified), KDA_ERR_INVALID_ARG when kda_chunk_fwd_varlen found bad
 * offsets, KDA_ERR_BOUNDS when (debug build only) an index check failed, or
 * KDA_ERR_CUDA when the synchronisation itself failed.
 *
 * Debug build.  libkda_debug.so is this library compiled with KDA_DEBUG: the
 * kernels check, before each access whose bounds rest on layout constants and
 * launch geometry (record indices and offsets, shared-memory tiles and tensor
 * operand views, token rows, state slices), that it stays in bounds; a failed
 * check skips the access and sets the status reported as KDA_ERR_BOUNDS.  It
 * exports the same symbols and is for testing; it is slower.
 */
KDA_API int kda_stream_status(void *stream);

/*
 * kda_chunk_fwd_debug_wait_limit -- test hook.  Sets the number of polls a
 * device-side wait makes before it gives up (0 restores the default, about
 * one second of polling).  A tiny limit lets a test exercise the timeout path
 * on a healthy GPU: the kernel records KDA_ERR_TIMEOUT, releases what it
 * holds and returns.  Applies to launches made after the call, process-wide.
 */
KDA_API void kda_chunk_fwd_debug_wait_limit(unsigned long long polls);

/*
 * kda_chunk_fwd_debug_inject_timeout -- test hook for the failure path.  When
 * `polls` is nonzero, every prefill CTA launched afterwards first waits (at
 * most `polls` polls, at most about one second) on a barrier that nothing
 * signals, gives up, records KDA_ERR_TIMEOUT, waits for its own copies in
 * flight, frees its tensor memory and returns without writing results.  The
 * GPU context stays usable.  0 turns the hook off.  Process-wide.
 */
KDA_API void kda_chunk_fwd_debug_inject_timeout(unsigned long long polls);

/*
 * kda_chunk_fwd_debug_force_exact -- test hook.  While enabled (enable != 0),
 * every chunk of every prefill launched afterwards takes the exact path that
 * otherwise only chunks with extreme decay take (see "Value domain" above), so
 * a test can compare the two paths on the same inputs.  Process-wide; off by
 * default.
 */
KDA_API void kda_chunk_fwd_debug_force_exact(int enable);

/*
 * kda_chunk_fwd_debug_block_refs -- test hook.  A chunk whose decay is mild
 * (every key channel's log-decay over the chunk >= -40) is normally formed
 * with one reference at the chunk's start; while enabled (enable != 0), every
 * chunk of every prefill launched afterwards is formed with the references of
 * its 16-token blocks instead, the form chunks with stronger decay take, so a
 * test can compare the two forms on the same inputs.  Process-wide; off by
 * default.
 */
KDA_API void kda_chunk_fwd_debug_block_refs(int enable);

/*
 * kda_chunk_fwd_debug_record_cap -- test hook.  Caps the bytes of chunk
 * records the prefill workspace holds at once (0 restores the default,
 * 2 GiB), so that small problems exercise the paths long ones take: segments
 * on two streams (kda_chunk_fwd) and windows (kda_chunk_fwd_varlen).
 * Applies to calls made afterwards; process-wide.
 */
KDA_API void kda_chunk_fwd_debug_record_cap(unsigned long long bytes);

/*
 * kda_chunk_fwd_debug_parts -- test hook for the two-level pass of
 * kda_chunk_fwd (long sequences with few (b, h)): 0 chooses the number of
 * parts per segment automatically (the default), 1 turns the two-level pass
 * off, P >= 3 forces P parts wherever a segment has at least P chunks.
 * Applies to calls made afterwards; process-wide.
 */
KDA_API void kda_chunk_fwd_debug_parts(int parts);

/*
 * kda_debug_kernel_timing -- measurement hook.  While enabled (enable != 0),
 * every kernel launch of the prefill and backward entry points gets a timing
 * slot: the kernel's own CTAs record, with %globaltimer, when the first of
 * them started and the last of them ended (two atomics per CTA; nothing is
 * added to the streams' ordering).  Kinds: 0 = the per-chunk prep kernel,
 * 1 = the state chain kernel, 2 = the exact kernel of steep chunks, 3 = the
 * two-level pass's fix-up, 4 = the backward pass (both of its kernels).
 * At most 8192 launches per device are timed between two reads.
 * Process-wide; off by default.
 *
 * kda_debug_kernel_times -- waits for the device(s), writes per kind the
 * summed busy time of the launches timed so far in ms (ms[kind]) and their
 * number (launches[kind]) for kinds < nkinds, and forgets them.  The host
 * arrays are the caller's.  KDA_OK, KDA_ERR_INVALID_ARG for NULL arrays, or
 * KDA_ERR_CUDA.
 */
KDA_API void kda_debug_kernel_timing(int enable);
KDA_API int kda_debug_kernel_times(double *ms, long long *launches, int nkinds);

/*
 * kda_debug_kernel_launches -- the same timed launches one by one, in the
 * order they were launched: kind[i], and start_ns[i] / end_ns[i], the
 * %globaltimer readings (nanoseconds, one clock per device) of the first CTA's
 * start and the last CTA's end; end_ns[i] < start_ns[i] for a launch that left
 * no stamp.  Writes at most `cap` entries (host arrays of the caller), the
 * number written to *count, and forgets every timed launch, like
 * kda_debug_kernel_times.  KDA_OK, KDA_ERR_INVALID_ARG for a NULL pointer or
 * cap < 0, or KDA_ERR_CUDA.
 */
KDA_API int kda_debug_kernel_launches(int *kind, long long *start_ns, long long *end_ns, int cap, int *count);

/* Version of this ABI (major * 100 + minor): 101 adds the scalar-gate entry
 * points, 102 the packed-batch prefill, the raw-input (fused gate prologue)
 * entry points, the backward pass and the exact-path and two-level test
 * hooks, 103 the host-buffer prefill and the per-launch timing list, 104 the
 * block-reference test hook. */
KDA_API int kda_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
