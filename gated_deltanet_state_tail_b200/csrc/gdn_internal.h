// gdn_internal.h -- structures shared by the host API and the kernels of the
// Tail-Replay library.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "gdn_tail_replay.h"

namespace gdn {

// Work window of one sequence, as validated on the host by the plan.
//   replay : rows [row0, row0 + len) are the tail of the matched prefix
//   prefill: rows [row0, row0 + len) are the whole sequence
// The expect_* fields are the descriptor values the window was derived from;
// kernels compare them with the device copies a caller passes.
struct Window {
    long long row0;
    int len;
    int expect_off;       // seq_offsets[b]
    int expect_end;       // seq_offsets[b + 1]
    int expect_match;     // replay: match_len[b]; prefill: unused
    int expect_budget;    // replay: R[b]; prefill: unused
    int pad;
};
static_assert(sizeof(Window) == 32, "Window is 32 bytes");

// One (sequence, head) work unit.  Plans order units longest first.
struct Unit {
    int seq;
    int head;
};

// Per-call device status at the start of the caller's workspace.  Nothing clears
// it between calls.  Each call carries a nonzero call number (CallArgs::epoch);
// every report tags a word with that number, dropping whatever an earlier number
// left in it, and the first thread of each launch records the number in `epoch`.
// A reader counts only the words whose tag equals that record (header_status), so
// no reset has to run on the stream ahead of the kernel.
struct WorkspaceHeader {
    unsigned long long status;  // (call number << 32) | kStatus* bits reported under it
    unsigned long long where;   // (call number << 32) | first wait that gave up (kernel-defined code)
    unsigned int epoch;         // call number of the last launch on this workspace
    unsigned int pad[59];
};
static_assert(sizeof(WorkspaceHeader) == 256, "header is 256 bytes");

constexpr unsigned int kStatusMismatch = 1u;
constexpr unsigned int kStatusTimeout = 2u;
constexpr unsigned int kStatusBounds = 4u;   // a checked index fell outside the plan (debug build)

// The kStatus* bits, and the first wait site that gave up, of the last call, from a
// header read back once the call is done.
__host__ __device__ inline unsigned int header_status(const WorkspaceHeader& h) {
    return (unsigned int)(h.status >> 32) == h.epoch ? (unsigned int)h.status : 0u;
}
__host__ __device__ inline unsigned int header_where(const WorkspaceHeader& h) {
    return (unsigned int)(h.where >> 32) == h.epoch ? (unsigned int)h.where : 0u;
}

// Next call number (never 0), for the host side of every entry point.
unsigned int next_call_number();

// Tags `word` with call number `epoch` and merges `val` into its low half: OR-ed in,
// or (first_only) stored only while the low half is still zero.  A retry follows
// another thread's change, and a word changes at most a few times per call (one
// retag, then once per status bit), so the loop ends; the cap only bounds it.  Out
// of line: inlined at every wait site, the loop slowed the prefill kernel by 3%.
static __device__ __noinline__ void tag_merge(unsigned long long* word, unsigned int epoch, unsigned int val,
                                          bool first_only) {
    unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(word);
    for (int i = 0; i < 64; ++i) {
        const unsigned int low = (unsigned int)(old >> 32) == epoch ? (unsigned int)old : 0u;
        const unsigned int nlow = first_only ? (low ? low : val) : (low | val);
        const unsigned long long want = ((unsigned long long)epoch << 32) | nlow;
        if (want == old) return;
        const unsigned long long seen = atomicCAS(word, old, want);
        if (seen == old) return;
        old = seen;
    }
}

// Index checks of the debug build (compiled with -DGDN_DEBUG_BOUNDS).  Each
// computed global row, head, column and state index is compared with the
// extents the plan validated on the host; a failing check sets kStatusBounds
// and the access is skipped (no trap, no out-of-range access).  In the release
// build every check is the constant `true` and compiles away.
#ifdef GDN_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
__device__ __forceinline__ bool index_ok(WorkspaceHeader* ws, unsigned int epoch, bool cond) {
    if (!cond) tag_merge(&ws->status, epoch, kStatusBounds, false);
    return cond;
}
#else
constexpr bool kDebugBounds = false;
__device__ __forceinline__ bool index_ok(WorkspaceHeader*, unsigned int, bool) { return true; }
#endif

// kFused: the replay window of each sequence, then its suffix with outputs, in one launch
enum PlanKind { kReplay = 0, kPrefill = 1, kFused = 2 };

// Everything a kernel needs for one call.
struct CallArgs {
    int kind;               // PlanKind
    int dtype;              // 0 = fp32, 1 = bf16 (q, k, v, o)
    int num_heads;
    int dk, dv;
    int batch;
    long long units;
    long long rows_total;   // rows of the packed buffers the plan addresses (max offset)
    long long rs_qk;        // elements between consecutive rows of q and k (H * dk when packed)
    long long rs_v;         // elements between consecutive rows of v (H * dv when packed)
    const Window* windows;  // [batch], plan-owned device memory
    const Unit* unit_list;  // [units], longest first
    // optional device descriptor arrays to check against the plan
    const int* chk_offsets; // [batch + 1] or null
    const int* chk_match;   // [batch] or null (replay)
    const int* chk_budget;  // [batch] or null (replay)
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;
    const float* beta;
    const float* state_in;  // null = zero state
    void* o_out;            // null = no outputs (the state-only replay)
    float* state_out;       // may be null for prefill
    WorkspaceHeader* ws;
    unsigned int epoch;     // this call's number (see WorkspaceHeader)
    // fused replay + suffix (chunked kernel): a first segment of rows per sequence,
    // replayed from the zero state without outputs before the rows of `windows`
    const Window* windows0; // [batch] or null
    long long rows_total0;  // rows of the buffers the first segment addresses
    const void* k0;
    const void* v0;
    const float* alpha0;
    const float* beta0;
    float* state_mid;       // null, or [batch, H, dk, dv]: the state after the first segment
    int replay_variant;     // ReplayVariant: which chunked kernel runs the state-only replay
};

// A status report of this call (see WorkspaceHeader).
__device__ __forceinline__ void report_status(const CallArgs& a, unsigned int bits) {
    tag_merge(&a.ws->status, a.epoch, bits, false);
}
__device__ __forceinline__ bool index_ok(const CallArgs& a, bool cond) { return index_ok(a.ws, a.epoch, cond); }
// The first thread of a launch records the call number; every kernel that takes a
// CallArgs does this before anything else.
__device__ __forceinline__ void record_call(const CallArgs& a) {
    if (blockIdx.x == 0 && threadIdx.x == 0) a.ws->epoch = a.epoch;
}

// The chunked path's state-only replay kernel: the two-CTA-per-SM kernel unless the
// descriptor's kernel field pins the warp-specialised or the cluster-pair one.
enum ReplayVariant { kReplayDefault = 0, kReplayTwoCta = 1, kReplayWarpSpec = 2, kReplayPair = 3 };

inline int replay_variant_of(int kernel) {
    return kernel == GDN_KERNEL_CHUNKED_TC_TWO_CTA    ? kReplayTwoCta
           : kernel == GDN_KERNEL_CHUNKED_TC_WARP_SPEC ? kReplayWarpSpec
           : kernel == GDN_KERNEL_CHUNKED_TC_PAIR      ? kReplayPair
                                                        : kReplayDefault;
}

// The kernel family a descriptor's kernel field names (the pinned replay variants
// are the chunked kernel).
inline int kernel_family_of(int kernel) {
    return (kernel == GDN_KERNEL_CHUNKED_TC_TWO_CTA || kernel == GDN_KERNEL_CHUNKED_TC_WARP_SPEC ||
            kernel == GDN_KERNEL_CHUNKED_TC_PAIR)
               ? GDN_KERNEL_CHUNKED_TC
               : kernel;
}

// Device-side check of one unit's window against the caller's descriptor
// arrays.  Returns true if the unit may run.
__device__ __forceinline__ bool window_agrees(const CallArgs& a, int b) {
    const Window& w = a.windows[b];
    if (a.chk_offsets) {
        if (a.chk_offsets[b] != w.expect_off || a.chk_offsets[b + 1] != w.expect_end) return false;
    }
    if (a.kind == kReplay) {
        if (a.chk_match && a.chk_match[b] != w.expect_match) return false;
        if (a.chk_budget && a.chk_budget[b] != w.expect_budget) return false;
    }
    return true;
}

// One decode step over a dense batch (no plan): q, k [batch, H, dk]; v, o
// [batch, H, dv]; alpha, beta [batch, H]; states [batch, H, dk, dv].
struct DecodeArgs {
    int dtype;              // 0 = fp32, 1 = bf16 (q, k, v, o)
    int num_heads;
    int dk, dv;
    long long batch;
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;
    const float* beta;
    const float* state_in;  // null = zero state
    float* state_out;       // may alias state_in; null = not written
    void* o_out;
};

// Raise a kernel's dynamic shared-memory limit once per device (a kernel attribute
// is per device); safe when several host threads launch at once.
inline cudaError_t ensure_smem_limit(const void* kernel, int bytes, std::atomic<uint64_t>& done_devices) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (done_devices.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done_devices.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// Host validation of a varlen descriptor shared by every entry point that takes
// one: sizes, dtype, kernel choice, offsets, row stride and the 64-bit extent bound.
gdn_status check_varlen_desc(const gdn_varlen_desc* d);

// Row strides (elements) of q/k and of v that a descriptor implies.
inline long long row_stride_qk(const gdn_varlen_desc* d) {
    return d->row_stride_elems ? d->row_stride_elems : (long long)d->num_heads * d->d_k;
}
inline long long row_stride_v(const gdn_varlen_desc* d) {
    return d->row_stride_elems ? d->row_stride_elems : (long long)d->num_heads * d->d_v;
}

cudaError_t launch_recurrent(const CallArgs& a, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_chunk_tc(const CallArgs& a, cudaStream_t stream);   // dispatches the replay below
cudaError_t launch_replay_tc(const CallArgs& a, cudaStream_t stream);
cudaError_t launch_replay_ws(const CallArgs& a, cudaStream_t stream);
cudaError_t launch_replay_pair(const CallArgs& a, cudaStream_t stream);
bool chunk_tc_supported(int dtype, int dk, int dv);

}  // namespace gdn
