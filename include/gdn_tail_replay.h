/*
 * gdn_tail_replay.h -- C ABI of the Tail-Replay state rebuild and chunked
 * suffix prefill for Gated DeltaNet layers on B200 (sm_100a).
 *
 * The method ("Tail-Replay: Escaping the Curse of Linear Attention in Prefix
 * Caching for Hybrid LLMs", gist.science summary, section "Mecanismos
 * Principais", item "Reconstrucao de Estado Independente"): on a prefix-cache
 * hit the recurrent state of each linear-attention (Gated DeltaNet) layer is
 * rebuilt by taking only the most recent R tokens of the matched prefix,
 * starting from a zero state, and replaying the layer's recurrence over that
 * tail.  The same page's "Resultados" section times the first token after
 * the hit, i.e. the prefill of the request's new suffix that continues from
 * the rebuilt state.
 *
 * The recurrence (Gated DeltaNet's gated delta rule), per head, with a
 * d_k x d_v state S whose rows are indexed by the key dimension:
 *     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 * alpha_t is the gate value in [0, 1] (not its log); no query scaling.
 *
 * Conventions shared by every call
 * --------------------------------
 *  Layout.  q, k: [rows, H, d_k]; v, o: [rows, H, d_v]; token-major rows,
 *    heads contiguous inside a row.  The rows of q, k and v are
 *    gdn_varlen_desc.row_stride_elems elements apart (0 = packed: H*d_k for
 *    q and k, H*d_v for v), so q, k and v may be slices of one fused
 *    projection buffer; o is always packed (row stride H*d_v).  alpha, beta:
 *    [rows, H] fp32 always (bf16 would round 0.999 to 1), packed.  States:
 *    [batch, H, d_k, d_v] fp32, row-major, key dimension first.
 *  dtype.  q, k, v and o share one element type: GDN_F32 or GDN_BF16.
 *  Ownership.  The caller owns every buffer.  The library allocates device
 *    memory only inside gdn_plan_create_* (a small schedule table) and frees
 *    it in gdn_plan_destroy.  No call on the hot path allocates.
 *  Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy
 *    default stream).  Every hot-path call is asynchronous on that stream.
 *  Errors.  Arguments are validated on the host before anything is
 *    launched; a rejected call launches nothing and returns a status.  Device
 *    code never traps: problems it detects (a descriptor array that disagrees
 *    with the plan, a wait that ran out) set bits in the workspace status
 *    word, which gdn_workspace_status() reads after the stream.
 *  Pointers.  Device buffers must be 16-byte aligned.
 *  Determinism.  Reruns on the same inputs give bit-identical results.
 *  Threads.  A plan is immutable after creation and may be used from
 *    several host threads; concurrent calls need separate workspaces.
 */
#ifndef GDN_TAIL_REPLAY_H
#define GDN_TAIL_REPLAY_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad offsets, misaligned buffer */
    GDN_ERR_UNSUPPORTED = 2,  /* head dims or dtype this build has no kernel for */
    GDN_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    GDN_ERR_TIMEOUT = 4,      /* a device-side wait gave up (reported via the workspace) */
    GDN_ERR_ALLOC = 5,        /* plan creation could not allocate */
    GDN_ERR_MISMATCH = 6,     /* device descriptor arrays disagree with the plan */
    GDN_ERR_BOUNDS = 7        /* debug build: a device index fell outside the plan's extents */
} gdn_status;

typedef enum gdn_dtype { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* Kernel selection.  AUTO picks the tensor-core chunked kernel for bf16 with
 * d_k = d_v = 128 and the exact fp32 CUDA-core recurrent kernel otherwise.
 * The chunked path has three state-only replay kernels: one with two CTAs per
 * SM (the one AUTO and GDN_KERNEL_CHUNKED_TC run), a warp-specialised one with
 * one CTA per SM, and a cluster-pair one that runs each (sequence, head) unit
 * on two CTAs on two SMs (one builds the chunks' T operands, the other runs
 * the state chain).  The values 3 to 5 pin one of them (for tests and
 * measurements); every other entry point treats them as
 * GDN_KERNEL_CHUNKED_TC. */
typedef enum gdn_kernel {
    GDN_KERNEL_AUTO = 0,
    GDN_KERNEL_RECURRENT = 1,              /* token-recurrent, fp32 CUDA cores, any supported shape */
    GDN_KERNEL_CHUNKED_TC = 2,             /* chunked WY/UT form on tcgen05 tensor cores (bf16, d = 128) */
    GDN_KERNEL_CHUNKED_TC_TWO_CTA = 3,     /* as 2, the replay always on the two-CTA-per-SM kernel */
    GDN_KERNEL_CHUNKED_TC_WARP_SPEC = 4,   /* as 2, the replay always on the warp-specialised kernel */
    GDN_KERNEL_CHUNKED_TC_PAIR = 5         /* as 2, the replay always on the cluster-pair kernel */
} gdn_kernel;

/* Varlen batch descriptor.  Sequence b occupies rows [seq_offsets[b],
 * seq_offsets[b+1]) of the row buffers.  Layer stacks are folded in by
 * treating (layer, request) pairs as sequences of one batch.
 * row_stride_elems: elements from one row of q, k or v to the next; 0 means
 * packed.  Otherwise it must be >= H * max(d_k, d_v) and a multiple of 16
 * bytes (8 bf16 or 4 fp32 elements: the tensor-core kernel reads rows with
 * TMA, whose strides are 16-byte multiples).  A fused [rows, 3, H, d]
 * projection buffer, for example, gives q, k and v with row stride 3*H*d.
 * rows * row stride must stay below 2^40 elements. */
typedef struct gdn_varlen_desc {
    int32_t batch;                    /* number of sequences, >= 1 */
    int32_t num_heads;                /* H, >= 1; batch * H <= 2^31 - 1 (one CTA per unit) */
    int32_t d_k;                      /* key head dim: 64 or 128 */
    int32_t d_v;                      /* value head dim: 64 or 128 */
    int32_t dtype;                    /* gdn_dtype of q, k, v, o */
    int32_t kernel;                   /* gdn_kernel; 0 = AUTO */
    const int32_t* seq_offsets_host;  /* [batch + 1] host copy; non-decreasing, [0] >= 0 */
    int64_t row_stride_elems;         /* q/k/v row stride in elements; 0 = packed */
} gdn_varlen_desc;

typedef struct gdn_plan* gdn_plan_t;

/*
 * Build the schedule of a tail replay ("Mecanismos Principais", item
 * "Reconstrucao de Estado Independente": the last k tokens of the matched
 * prefix, replayed from a zero state).
 *   cache          descriptor of the prefix cache rows; the cached entry of
 *                  sequence b may be longer than its match.
 *   match_len_host [batch] matched prefix length L_b, 0 <= L_b <= cached length.
 *   R_host         [batch] replay budget R_b >= 0; R_b > L_b is clamped to L_b,
 *                  R_b = 0 (or L_b = 0) yields the zero state ("Zero-Only").
 * Sequence b's window is rows [off_b + L_b - min(R_b, L_b), off_b + L_b).
 * The plan copies what it needs; the host arrays may be freed afterwards.
 * Returns GDN_OK, INVALID_ARG, UNSUPPORTED, ALLOC or CUDA.
 */
GDN_API gdn_status gdn_plan_create_replay(const gdn_varlen_desc* cache, const int32_t* match_len_host,
                                  const int32_t* R_host, gdn_plan_t* out);

/*
 * Build the schedule of a chunked prefill over whole sequences (the suffix
 * prefill that follows the rebuild, "Resultados" section: time to first
 * token; with a zero initial state over prefix ++ suffix it is the full
 * prefill the pages compare against).  Sequence b is rows [off_b, off_b+1).
 */
GDN_API gdn_status gdn_plan_create_prefill(const gdn_varlen_desc* seqs, gdn_plan_t* out);

/*
 * Build the schedule of a fused rebuild + suffix prefill: for each sequence,
 * the replay window of gdn_plan_create_replay (from a zero state, no
 * outputs), then the sequence's new suffix with outputs, continuing from the
 * replayed state (the pages' cache hit: "Mecanismos Principais" rebuilds the
 * state, "Resultados" times the suffix prefill that follows).
 *   cache, match_len_host, R_host   as for gdn_plan_create_replay.
 *   suffix_offsets_host             [batch + 1] row offsets of the suffixes in
 *                                   their own row buffers (non-decreasing).
 * The suffix buffers share the cache descriptor's heads, dims, dtype, row
 * stride and kernel choice.  gdn_plan_window reports the replay window.
 */
GDN_API gdn_status gdn_plan_create_fused(const gdn_varlen_desc* cache, const int32_t* match_len_host,
                                         const int32_t* R_host, const int32_t* suffix_offsets_host,
                                         gdn_plan_t* out);

/* The replay windows a replay plan would use, computed on the host with no
 * device work: row0_out[b] = seq_offsets[b] + L_b - min(R_b, L_b) and
 * len_out[b] = min(R_b, L_b).  Same validation as gdn_plan_create_replay
 * (INVALID_ARG for a match longer than its cached entry, R_b < 0, offsets
 * that decrease, or null pointers); nothing is written on error. */
GDN_API gdn_status gdn_replay_windows(int32_t batch, const int32_t* seq_offsets_host,
                                      const int32_t* match_len_host, const int32_t* R_host,
                                      int64_t* row0_out, int32_t* len_out);

/* Free a plan (NULL is ignored).  Synchronises with nothing; do not destroy a
 * plan while a call that uses it may still be running. */
GDN_API void gdn_plan_destroy(gdn_plan_t plan);

/* First row and length of sequence b's work window (replay and fused: the
 * tail window; prefill: the whole sequence).  For tests and schedulers. */
GDN_API gdn_status gdn_plan_window(gdn_plan_t plan, int32_t b, int64_t* row0, int32_t* len);

/* Number of (sequence, head) work units and the kernel the plan will run. */
GDN_API gdn_status gdn_plan_info(gdn_plan_t plan, int64_t* units, int64_t* total_tokens,
                         int32_t* kernel);

/* Kernel launches that one call on this plan makes: 1 for a replay or a
 * prefill plan; 1 or 2 for a fused plan (see gdn_tail_replay_prefill).  A
 * call puts nothing else on its stream.  INVALID_ARG for a NULL plan or
 * pointer. */
GDN_API gdn_status gdn_plan_launches(gdn_plan_t plan, int32_t* launches);

/* Bytes of device workspace a call on this plan needs (>= 256, multiple of
 * 256).  The caller allocates it (16-byte aligned) and passes it to each
 * call; calls running concurrently need separate workspaces.  Its contents
 * need no initialisation and no reset between calls: each call tags the
 * status it reports with a call number of its own, and the call's first
 * thread records that number, so gdn_workspace_status reads only what the
 * last call reported. */
GDN_API size_t gdn_workspace_bytes(gdn_plan_t plan);

/*
 * Tail replay: rebuild the state at the end of each matched prefix.
 *   q            unused by the state-only replay; may be NULL.
 *   k, v         cache rows (row stride of the plan), dtype of the plan.
 *   alpha, beta  [rows, H] fp32 gates of the cached rows.
 *   seq_offsets, match_len, R
 *                device copies of the arrays given to the plan ([batch+1],
 *                [batch], [batch] int32), or NULL.  When given, each work
 *                unit checks its window against them; a disagreement skips
 *                the unit and sets GDN_ERR_MISMATCH in the workspace.
 *                Addressing always uses the plan's validated copy.
 *   state_out    [batch, H, d_k, d_v] fp32, written in full.
 *   workspace    gdn_workspace_bytes(plan) bytes of device memory.
 *   stream       cudaStream_t.
 * Host-side return: GDN_OK or an argument/launch error.  Device-side
 * problems are read with gdn_workspace_status().
 */
GDN_API gdn_status gdn_tail_replay_state(gdn_plan_t plan, const void* q, const void* k, const void* v,
                                 const float* alpha, const float* beta,
                                 const int32_t* seq_offsets, const int32_t* match_len,
                                 const int32_t* R, float* state_out, void* workspace,
                                 void* stream);

/*
 * Tail replay that also emits the replayed tokens' outputs: for every row t
 * of sequence b's window, o_t = S_t^T q_t with S the state replayed from
 * zero since the window's first row (the same states gdn_tail_replay_state
 * rebuilds).  Within a group of GDN layers that Tail-Replay replays together
 * ("Mecanismos Principais", item "Reconstrucao de Estado Independente": each
 * group after a full-attention layer is rebuilt independently), these are
 * the outputs a layer hands to the next one.
 *   q            [rows, H, d_k] with the row stride of k; required.
 *   k, v, alpha, beta, seq_offsets, match_len, R
 *                as for gdn_tail_replay_state.
 *   o_out        [rows, H, d_v] in the plan's dtype, addressed like q: the
 *                window rows are written, every other row is left untouched.
 *   state_out    [batch, H, d_k, d_v] fp32, or NULL.
 * It runs the output-writing kernels (the prefill ones, from a zero state),
 * so it costs a prefill of the window rather than a state-only replay.
 * Returns as gdn_tail_replay_state; INVALID_ARG for a prefill plan or a NULL
 * o_out.
 */
GDN_API gdn_status gdn_tail_replay_outputs(gdn_plan_t plan, const void* q, const void* k, const void* v,
                                           const float* alpha, const float* beta,
                                           const int32_t* seq_offsets, const int32_t* match_len,
                                           const int32_t* R, void* o_out, float* state_out,
                                           void* workspace, void* stream);

/*
 * One decode step (the token after the prefill; the pages time the first
 * one as TTFT, "Resultados"), for a dense batch with no plan:
 *   S' = alpha (I - beta k k^T) S + beta k v^T,   o = S'^T q.
 *   batch, num_heads, d_k, d_v, dtype
 *                sizes (d in {64, 128}) and the element type of q, k, v, o.
 *   q, k         [batch, H, d_k];  v, o_out: [batch, H, d_v]  (dtype).
 *   alpha, beta  [batch, H] fp32.
 *   state_in     [batch, H, d_k, d_v] fp32, or NULL for the zero state.
 *   state_out    [batch, H, d_k, d_v] fp32, or NULL; may equal state_in
 *                (updated in place).
 *   stream       cudaStream_t.
 * The step waits on nothing on the device, so it has no workspace and no
 * device status.  batch = 0 launches nothing.  Returns GDN_OK,
 * INVALID_ARG (null or misaligned pointers, batch < 0, H < 1), UNSUPPORTED
 * (head dims or dtype) or CUDA.
 */
GDN_API gdn_status gdn_decode_step(int32_t batch, int32_t num_heads, int32_t d_k, int32_t d_v,
                                   int32_t dtype, const void* q, const void* k, const void* v,
                                   const float* alpha, const float* beta, const float* state_in,
                                   float* state_out, void* o_out, void* stream);

/*
 * Chunked prefill over each sequence of a prefill plan, continuing from
 * state_in, emitting o_t = S_t^T q_t for every row and the final state.
 *   q, k, v      rows (row stride of the plan), dtype of the plan.
 *   alpha, beta  [rows, H] fp32.
 *   cu_seqlens   device copy of the plan's offsets ([batch+1] int32) or NULL;
 *                checked like the replay's descriptor arrays.
 *   state_in     [batch, H, d_k, d_v] fp32, or NULL for the zero state.
 *   o_out        [rows, H, d_v] in the plan's dtype; rows of the sequences
 *                are written, other rows are left untouched.
 *   state_out    [batch, H, d_k, d_v] fp32, or NULL.  May alias state_in.
 */
GDN_API gdn_status gdn_chunk_prefill(gdn_plan_t plan, const void* q, const void* k, const void* v,
                             const float* alpha, const float* beta, const int32_t* cu_seqlens,
                             const float* state_in, void* o_out, float* state_out,
                             void* workspace, void* stream);

/*
 * Fused rebuild + suffix prefill on a fused plan: equal (up to rounding
 * order) to gdn_tail_replay_state followed by gdn_chunk_prefill from the
 * rebuilt states.  The plan fixes how it runs.  On the tensor-core kernel,
 * when no replay window is longer than 320 tokens, or when the plan has no
 * more (sequence, head) units than the GPU has SMs and no window is longer
 * than 1024 tokens, it is one launch and the state stays on chip between
 * the two phases.  Otherwise, on that kernel
 * with a replay kernel pinned, and on the fp32 recurrent kernel, it is a
 * state-only replay launch writing state_mid (or state_out) and a prefill
 * launch reading it back: longer windows replay faster on the replay
 * kernel than inside the one-launch kernel.  gdn_plan_launches tells which.
 *   k, v, alpha, beta        the cache rows (as for the replay).
 *   sq, sk, sv, salpha, sbeta
 *                            the suffix rows (as for the prefill).
 *   o_out                    [suffix rows, H, d_v] plan dtype; suffix rows written.
 *   state_mid                [batch, H, d_k, d_v] fp32 or NULL: the rebuilt state
 *                            at the end of the matched prefix.
 *   state_out                [batch, H, d_k, d_v] fp32: the state after the suffix.
 * No device descriptor arrays are checked.  Returns as gdn_chunk_prefill;
 * INVALID_ARG for a plan that is not fused or a NULL state_out.
 */
GDN_API gdn_status gdn_tail_replay_prefill(gdn_plan_t plan, const void* k, const void* v,
                                           const float* alpha, const float* beta, const void* sq,
                                           const void* sk, const void* sv, const float* salpha,
                                           const float* sbeta, void* o_out, float* state_mid,
                                           float* state_out, void* workspace, void* stream);

/*
 * Tail replay that allocates nothing (the pages describe no counterpart; this
 * is a deployment variant of gdn_tail_replay_state).
 *
 * For callers that cannot call cudaMalloc -- code running inside a memory
 * pool that owns the whole device heap, or a runtime that only hands out its
 * own input and output buffers -- and so can neither create a plan (its
 * schedule table is device memory) nor provide a workspace.  The schedule
 * and the status word live in one fixed 64 KB __device__ array inside the
 * library, which every GPU that loads the library holds until the process
 * exits.  The call validates like gdn_plan_create_replay, builds the
 * schedule in a per-thread static host buffer (not on the caller's stack),
 * copies it into that array on `stream`, clears the status word and
 * launches the same kernel a plan would.  No cudaMalloc, cudaFree or other
 * allocating routine is called.
 *   cache, match_len_host, R_host   as for gdn_plan_create_replay.
 *   k, v, alpha, beta, state_out    as for gdn_tail_replay_state.
 *   stream                          cudaStream_t.
 *   status_out                      NULL, or a host word that receives the
 *                                   device status (0 = ok, else the bit set
 *                                   gdn_workspace_status decodes); the call
 *                                   then waits for `stream`.
 * Limit: 256 + 32 * batch + 8 * batch * num_heads bytes (plus 16 * batch of
 * host temporaries) must fit in 64 KB; larger batches return
 * GDN_ERR_UNSUPPORTED before anything is launched.
 * Every call looks up the array's device address on the current device
 * (so a recreated context is handled); the first call on a device also loads
 * the library's device code there, so make that first call before any stream
 * capture.  Every call on a device shares the array, which keeps the last
 * call's contents, so calls whose work overlaps on the GPU (different
 * streams, or several host threads) race.
 */
GDN_API gdn_status gdn_tail_replay_state_noalloc(const gdn_varlen_desc* cache,
                                                 const int32_t* match_len_host,
                                                 const int32_t* R_host, const void* k,
                                                 const void* v, const float* alpha,
                                                 const float* beta, float* state_out,
                                                 void* stream, uint32_t* status_out);

/* Synchronise `stream`, then return the status the device recorded in
 * `workspace` during the last call (GDN_OK, GDN_ERR_TIMEOUT, GDN_ERR_BOUNDS
 * or GDN_ERR_MISMATCH, in that order of precedence), or GDN_ERR_CUDA if the
 * stream itself failed. */
GDN_API gdn_status gdn_workspace_status(const void* workspace, void* stream);

/*
 * Self-test of the failure path (the pages describe no counterpart).  Every
 * kernel bounds its device waits; one that runs out records GDN_ERR_TIMEOUT
 * and the wait site in the workspace and returns, so the context stays usable.
 * This launches one thread that waits, for limit_ns nanoseconds (1 .. 1e9),
 * on an mbarrier that nothing arrives on.  Afterwards gdn_workspace_status()
 * returns GDN_ERR_TIMEOUT and the next call on the context works as usual.
 *   workspace   >= 256 bytes of device memory, 16-byte aligned (its header
 *               is cleared first).
 * Returns GDN_OK, INVALID_ARG or CUDA.
 */
GDN_API gdn_status gdn_selftest_bounded_wait(uint64_t limit_ns, void* workspace, void* stream);

/*
 * Test aid for callers' failure paths (the pages describe no counterpart):
 * the next `count` plan creations in this process (gdn_plan_create_*) fail
 * with GDN_ERR_ALLOC at the point where they would allocate their device
 * schedule table, before any device call, and free what they built on the
 * host.  count <= 0 clears a pending injection.  Thread-safe; meant for
 * tests, so that an out-of-memory path can be exercised without exhausting
 * the device.
 */
GDN_API void gdn_debug_fail_plan_allocations(int32_t count);

/*
 * Debug build (libgdn_tail_replay_debug.so, compiled with -DGDN_DEBUG_BOUNDS;
 * the pages describe no counterpart).  Every kernel that has a workspace
 * checks each global row, head, column and state index it computes against
 * the extents the plan validated on the host.  A failing check skips the
 * access and sets GDN_ERR_BOUNDS in the workspace status; nothing traps.
 * The decode step has no workspace: its indices come from its grid alone.
 * gdn_debug_bounds_enabled() returns 1 in the debug build, 0 otherwise.
 * gdn_selftest_index_check() runs one failing check (on an index one past a
 * 4-element extent, access skipped) so that gdn_workspace_status() then
 * returns GDN_ERR_BOUNDS; the release build returns GDN_ERR_UNSUPPORTED.
 *   workspace   >= 256 bytes of device memory, 16-byte aligned (cleared first).
 */
GDN_API int32_t gdn_debug_bounds_enabled(void);
GDN_API gdn_status gdn_selftest_index_check(void* workspace, void* stream);

/* Static description of a status code. */
GDN_API const char* gdn_status_string(gdn_status s);

/* Library version (major * 10000 + minor * 100 + patch). */
GDN_API int32_t gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_TAIL_REPLAY_H */
