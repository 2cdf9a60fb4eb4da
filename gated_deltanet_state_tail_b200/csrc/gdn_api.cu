// gdn_api.cu -- host side of the Tail-Replay C ABI: argument validation, the
// varlen plan (windows, work units, longest-first order) and kernel dispatch.
//
// The replay window follows "Tail-Replay: Escaping the Curse of Linear
// Attention in Prefix Caching for Hybrid LLMs", section "Mecanismos
// Principais", item "Reconstrucao de Estado Independente": only the most
// recent R tokens of the matched prefix are replayed, from a zero state.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "gdn_internal.h"
#include "gdn_tail_replay.h"

using gdn::CallArgs;
using gdn::Unit;
using gdn::Window;
using gdn::WorkspaceHeader;

struct gdn_plan {
    int kind;
    int batch, num_heads, dk, dv, dtype, kernel;
    int replay_variant;       // gdn::ReplayVariant (chunked kernel, state-only replay)
    bool fused_one_launch;    // fused plan, chunked kernel: the windows and the suffix in one launch
    long long rs_qk, rs_v;    // row strides (elements) of q/k and of v
    int device;
    std::vector<Window> windows;   // replay: the tail windows; prefill and fused: the (suffix) sequences
    std::vector<Window> windows0;  // fused: the replay windows run before `windows`
    std::vector<Unit> units;
    long long total_tokens;
    long long rows_total;     // rows the windows address (max end offset)
    long long rows_total0;    // fused: rows the replay windows address
    void* dev_block;          // windows, windows0, then units
    Window* d_windows;
    Window* d_windows0;
    Unit* d_units;
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace gdn {

unsigned int next_call_number() {
    static std::atomic<unsigned int> counter{0};
    unsigned int n = counter.fetch_add(1, std::memory_order_relaxed) + 1;
    while (n == 0) n = counter.fetch_add(1, std::memory_order_relaxed) + 1;   // 0 is never a call number
    return n;
}

gdn_status check_varlen_desc(const gdn_varlen_desc* d) {
    if (!d || !d->seq_offsets_host) return GDN_ERR_INVALID_ARG;
    if (d->batch < 1 || d->num_heads < 1) return GDN_ERR_INVALID_ARG;
    if (d->dtype != GDN_F32 && d->dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if ((d->d_k != 64 && d->d_k != 128) || (d->d_v != 64 && d->d_v != 128)) return GDN_ERR_UNSUPPORTED;
    if (d->kernel < GDN_KERNEL_AUTO || d->kernel > GDN_KERNEL_CHUNKED_TC_PAIR) return GDN_ERR_INVALID_ARG;
    // row stride: 0 = packed; otherwise every head of a row fits and rows start on 16 bytes
    if (d->row_stride_elems != 0) {
        const long long elem = d->dtype == GDN_BF16 ? 2 : 4;
        const long long widest = (long long)d->num_heads * (d->d_k > d->d_v ? d->d_k : d->d_v);
        if (d->row_stride_elems < widest || (d->row_stride_elems * elem) % 16 != 0) return GDN_ERR_INVALID_ARG;
        if (d->row_stride_elems > (1ll << 40)) return GDN_ERR_INVALID_ARG;
    }
    const int32_t* off = d->seq_offsets_host;
    if (off[0] < 0) return GDN_ERR_INVALID_ARG;
    for (int b = 0; b < d->batch; ++b)
        if (off[b + 1] < off[b]) return GDN_ERR_INVALID_ARG;
    // element offsets are 64-bit on the device; rows * row stride must fit comfortably
    const long long rows = off[d->batch];
    const long long rs = row_stride_qk(d) > row_stride_v(d) ? row_stride_qk(d) : row_stride_v(d);
    if (rows * d->num_heads > (1ll << 40) || rows * rs > (1ll << 46)) return GDN_ERR_INVALID_ARG;
    // one CTA per (sequence, head) unit: the unit count is the grid's x extent
    if ((long long)d->batch * d->num_heads > 0x7fffffffll) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

}  // namespace gdn

namespace {

gdn_status check_desc(const gdn_varlen_desc* d) { return gdn::check_varlen_desc(d); }

// Plan creations still to fail with GDN_ERR_ALLOC (gdn_debug_fail_plan_allocations).
std::atomic<int> g_fail_plan_allocs{0};

bool take_injected_alloc_failure() {
    int pending = g_fail_plan_allocs.load(std::memory_order_relaxed);
    while (pending > 0 && !g_fail_plan_allocs.compare_exchange_weak(pending, pending - 1)) {
    }
    return pending > 0;
}

int resolve_kernel(const gdn_varlen_desc* d) {
    if (d->kernel != GDN_KERNEL_AUTO) return gdn::kernel_family_of(d->kernel);
    return gdn::chunk_tc_supported(d->dtype, d->d_k, d->d_v) ? GDN_KERNEL_CHUNKED_TC
                                                              : GDN_KERNEL_RECURRENT;
}

// Longest replay windows (tokens) that a fused call on the chunked kernel still runs as one
// launch.  One launch keeps the state on chip between the window and the suffix and saves a
// launch, but its window chunks run on the one-CTA-per-SM prefill kernel, slower per chunk
// than the two-CTA state-only replay kernel.  Measured on B200 (bf16, d = 128, 512-token
// suffix): with at most one unit per SM, one launch is 2-12 us faster up to 13 chunks, within
// 2 us either way at 20 and up to 28 us slower at 52; with 192 to 444 units, 2-18 us faster
// up to 5 chunks and 3.5-5 us slower at 7.
constexpr int kFusedOneLaunchMaxTokens = 16 * 64;         // at most one unit per SM
constexpr int kFusedOneLaunchMaxTokensAnyUnits = 5 * 64;  // any number of units

// A fused plan on the chunked kernel runs as one launch when no window is longer than
// kFusedOneLaunchMaxTokensAnyUnits, or when every (sequence, head) unit has an SM of its own
// and no window is longer than kFusedOneLaunchMaxTokens; otherwise as the state-only replay
// launch followed by the prefill launch.  A descriptor that pins a replay kernel always takes
// the two launches.
gdn_status choose_fused_schedule(gdn_plan* p) {
    p->fused_one_launch = false;
    if (p->kernel != GDN_KERNEL_CHUNKED_TC || p->replay_variant != gdn::kReplayDefault) return GDN_OK;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, p->device) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_CUDA;
    }
    int longest = 0;
    for (const Window& w : p->windows0) longest = std::max(longest, (int)w.len);
    p->fused_one_launch = longest <= kFusedOneLaunchMaxTokensAnyUnits ||
                          ((long long)p->batch * p->num_heads <= sms && longest <= kFusedOneLaunchMaxTokens);
    return GDN_OK;
}

gdn_status finish_plan(gdn_plan* p, gdn_plan_t* out) {
    // Work units: every (sequence, head); longest window first so the long
    // units start early and the short ones fill the tail of the grid.
    p->units.reserve((size_t)p->batch * p->num_heads);
    for (int b = 0; b < p->batch; ++b)
        for (int h = 0; h < p->num_heads; ++h) p->units.push_back(Unit{b, h});
    auto unit_len = [p](int b) {
        return (long long)p->windows[b].len + (p->windows0.empty() ? 0 : p->windows0[b].len);
    };
    std::stable_sort(p->units.begin(), p->units.end(),
                     [&unit_len](const Unit& x, const Unit& y) { return unit_len(x.seq) > unit_len(y.seq); });
    p->total_tokens = 0;
    p->rows_total = 0;
    p->rows_total0 = 0;
    for (const Window& w : p->windows) {
        p->total_tokens += w.len;
        p->rows_total = std::max(p->rows_total, (long long)w.expect_end);
    }
    for (const Window& w : p->windows0) {
        p->total_tokens += w.len;
        p->rows_total0 = std::max(p->rows_total0, (long long)w.expect_end);
    }

    // an injected failure stands where the device allocation would fail
    if (take_injected_alloc_failure()) return GDN_ERR_ALLOC;
    if (cudaGetDevice(&p->device) != cudaSuccess) return GDN_ERR_CUDA;
    if (p->kind == gdn::kFused) {
        const gdn_status s = choose_fused_schedule(p);
        if (s != GDN_OK) return s;
    }
    const size_t wbytes = sizeof(Window) * p->windows.size();
    const size_t w0bytes = sizeof(Window) * p->windows0.size();
    const size_t ubytes = sizeof(Unit) * p->units.size();
    if (cudaMalloc(&p->dev_block, wbytes + w0bytes + ubytes) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_ALLOC;
    }
    p->d_windows = static_cast<Window*>(p->dev_block);
    p->d_windows0 = w0bytes ? reinterpret_cast<Window*>(static_cast<char*>(p->dev_block) + wbytes) : nullptr;
    p->d_units = reinterpret_cast<Unit*>(static_cast<char*>(p->dev_block) + wbytes + w0bytes);
    if (cudaMemcpy(p->d_windows, p->windows.data(), wbytes, cudaMemcpyHostToDevice) != cudaSuccess ||
        (w0bytes && cudaMemcpy(p->d_windows0, p->windows0.data(), w0bytes, cudaMemcpyHostToDevice) != cudaSuccess) ||
        cudaMemcpy(p->d_units, p->units.data(), ubytes, cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaFree(p->dev_block);
        p->dev_block = nullptr;
        return GDN_ERR_CUDA;
    }
    *out = p;
    return GDN_OK;
}

gdn_status check_replay_arrays(int batch, const int32_t* off, const int32_t* match_len,
                               const int32_t* R) {
    if (batch < 1 || !off || !match_len || !R) return GDN_ERR_INVALID_ARG;
    if (off[0] < 0) return GDN_ERR_INVALID_ARG;
    for (int b = 0; b < batch; ++b) {
        const long long cached = (long long)off[b + 1] - off[b];
        if (cached < 0) return GDN_ERR_INVALID_ARG;
        if (match_len[b] < 0 || match_len[b] > cached) return GDN_ERR_INVALID_ARG;
        if (R[b] < 0) return GDN_ERR_INVALID_ARG;
    }
    return GDN_OK;
}

gdn_plan* new_plan(const gdn_varlen_desc* d, int kind) {
    gdn_plan* p = new (std::nothrow) gdn_plan();
    if (!p) return nullptr;
    p->kind = kind;
    p->batch = d->batch;
    p->num_heads = d->num_heads;
    p->dk = d->d_k;
    p->dv = d->d_v;
    p->dtype = d->dtype;
    p->kernel = resolve_kernel(d);
    p->replay_variant = gdn::replay_variant_of(d->kernel);
    p->rs_qk = gdn::row_stride_qk(d);
    p->rs_v = gdn::row_stride_v(d);
    p->fused_one_launch = false;
    p->dev_block = nullptr;
    p->d_windows0 = nullptr;
    return p;
}

void fill_replay_windows(std::vector<Window>& win, int batch, const int32_t* off, const int32_t* match_len,
                         const int32_t* R) {
    win.resize(batch);
    std::vector<int64_t> row0(batch);
    std::vector<int32_t> len(batch);
    gdn_replay_windows(batch, off, match_len, R, row0.data(), len.data());
    for (int b = 0; b < batch; ++b) {
        Window& w = win[b];
        std::memset(&w, 0, sizeof w);
        w.row0 = row0[b];   // R > L clamps to L; R = 0 is the Zero-Only state
        w.len = len[b];
        w.expect_off = off[b];
        w.expect_end = off[b + 1];
        w.expect_match = match_len[b];
        w.expect_budget = R[b];
    }
}

void fill_sequence_windows(std::vector<Window>& win, int batch, const int32_t* off) {
    win.resize(batch);
    for (int b = 0; b < batch; ++b) {
        Window& w = win[b];
        std::memset(&w, 0, sizeof w);
        w.row0 = off[b];
        w.len = off[b + 1] - off[b];
        w.expect_off = off[b];
        w.expect_end = off[b + 1];
    }
}

gdn_status check_call_common(gdn_plan_t plan, void* workspace) {
    if (!plan || !workspace) return GDN_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return GDN_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (dev != plan->device) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

gdn_status launch(gdn_plan_t plan, CallArgs& a, cudaStream_t stream) {
    cudaError_t e = plan->kernel == GDN_KERNEL_CHUNKED_TC ? gdn::launch_chunk_tc(a, stream)
                                                          : gdn::launch_recurrent(a, stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_CUDA;
    }
    return GDN_OK;
}

void fill_common(gdn_plan_t plan, CallArgs& a, void* workspace) {
    a.kind = plan->kind;
    a.dtype = plan->dtype;
    a.num_heads = plan->num_heads;
    a.dk = plan->dk;
    a.dv = plan->dv;
    a.batch = plan->batch;
    a.units = (long long)plan->units.size();
    a.rows_total = plan->rows_total;
    a.rs_qk = plan->rs_qk;
    a.rs_v = plan->rs_v;
    a.windows = plan->d_windows;
    a.unit_list = plan->d_units;
    a.ws = static_cast<WorkspaceHeader*>(workspace);
    a.epoch = gdn::next_call_number();
    a.replay_variant = plan->replay_variant;
}

}  // namespace

extern "C" {

gdn_status gdn_plan_create_replay(const gdn_varlen_desc* cache, const int32_t* match_len_host,
                                  const int32_t* R_host, gdn_plan_t* out) {
    if (!out) return GDN_ERR_INVALID_ARG;
    *out = nullptr;
    gdn_status s = check_desc(cache);
    if (s != GDN_OK) return s;
    if (!match_len_host || !R_host) return GDN_ERR_INVALID_ARG;
    const int32_t* off = cache->seq_offsets_host;
    s = check_replay_arrays(cache->batch, off, match_len_host, R_host);
    if (s != GDN_OK) return s;
    if (resolve_kernel(cache) == GDN_KERNEL_CHUNKED_TC &&
        !gdn::chunk_tc_supported(cache->dtype, cache->d_k, cache->d_v))
        return GDN_ERR_UNSUPPORTED;
    gdn_plan* p = new_plan(cache, gdn::kReplay);
    if (!p) return GDN_ERR_ALLOC;
    try {   // host allocations report GDN_ERR_ALLOC instead of throwing across the C ABI
        fill_replay_windows(p->windows, cache->batch, off, match_len_host, R_host);
        s = finish_plan(p, out);
    } catch (const std::bad_alloc&) {
        s = GDN_ERR_ALLOC;
    }
    if (s != GDN_OK) delete p;
    return s;
}

gdn_status gdn_plan_create_prefill(const gdn_varlen_desc* seqs, gdn_plan_t* out) {
    if (!out) return GDN_ERR_INVALID_ARG;
    *out = nullptr;
    gdn_status s = check_desc(seqs);
    if (s != GDN_OK) return s;
    if (resolve_kernel(seqs) == GDN_KERNEL_CHUNKED_TC &&
        !gdn::chunk_tc_supported(seqs->dtype, seqs->d_k, seqs->d_v))
        return GDN_ERR_UNSUPPORTED;
    gdn_plan* p = new_plan(seqs, gdn::kPrefill);
    if (!p) return GDN_ERR_ALLOC;
    try {
        fill_sequence_windows(p->windows, seqs->batch, seqs->seq_offsets_host);
        s = finish_plan(p, out);
    } catch (const std::bad_alloc&) {
        s = GDN_ERR_ALLOC;
    }
    if (s != GDN_OK) delete p;
    return s;
}

gdn_status gdn_plan_create_fused(const gdn_varlen_desc* cache, const int32_t* match_len_host,
                                 const int32_t* R_host, const int32_t* suffix_offsets_host, gdn_plan_t* out) {
    if (!out) return GDN_ERR_INVALID_ARG;
    *out = nullptr;
    gdn_status s = check_desc(cache);
    if (s != GDN_OK) return s;
    if (!match_len_host || !R_host || !suffix_offsets_host) return GDN_ERR_INVALID_ARG;
    const int32_t* off = cache->seq_offsets_host;
    s = check_replay_arrays(cache->batch, off, match_len_host, R_host);
    if (s != GDN_OK) return s;
    gdn_varlen_desc suf = *cache;   // same batch, heads, dims, dtype and kernel; suffix offsets
    suf.seq_offsets_host = suffix_offsets_host;
    s = check_desc(&suf);
    if (s != GDN_OK) return s;
    if (resolve_kernel(cache) == GDN_KERNEL_CHUNKED_TC &&
        !gdn::chunk_tc_supported(cache->dtype, cache->d_k, cache->d_v))
        return GDN_ERR_UNSUPPORTED;
    gdn_plan* p = new_plan(cache, gdn::kFused);
    if (!p) return GDN_ERR_ALLOC;
    try {
        fill_replay_windows(p->windows0, cache->batch, off, match_len_host, R_host);
        fill_sequence_windows(p->windows, cache->batch, suffix_offsets_host);
        s = finish_plan(p, out);
    } catch (const std::bad_alloc&) {
        s = GDN_ERR_ALLOC;
    }
    if (s != GDN_OK) delete p;
    return s;
}

gdn_status gdn_replay_windows(int32_t batch, const int32_t* seq_offsets_host,
                              const int32_t* match_len_host, const int32_t* R_host,
                              int64_t* row0_out, int32_t* len_out) {
    if (!row0_out || !len_out) return GDN_ERR_INVALID_ARG;
    gdn_status s = check_replay_arrays(batch, seq_offsets_host, match_len_host, R_host);
    if (s != GDN_OK) return s;
    for (int b = 0; b < batch; ++b) {
        const int L = match_len_host[b];
        const int reff = std::min(R_host[b], L);
        row0_out[b] = (int64_t)seq_offsets_host[b] + L - reff;
        len_out[b] = reff;
    }
    return GDN_OK;
}

void gdn_plan_destroy(gdn_plan_t plan) {
    if (!plan) return;
    if (plan->dev_block) cudaFree(plan->dev_block);
    delete plan;
}

gdn_status gdn_plan_window(gdn_plan_t plan, int32_t b, int64_t* row0, int32_t* len) {
    if (!plan || !row0 || !len || b < 0 || b >= plan->batch) return GDN_ERR_INVALID_ARG;
    const Window& w = plan->kind == gdn::kFused ? plan->windows0[b] : plan->windows[b];
    *row0 = w.row0;
    *len = w.len;
    return GDN_OK;
}

gdn_status gdn_plan_info(gdn_plan_t plan, int64_t* units, int64_t* total_tokens, int32_t* kernel) {
    if (!plan) return GDN_ERR_INVALID_ARG;
    if (units) *units = (int64_t)plan->units.size();
    if (total_tokens) *total_tokens = plan->total_tokens;
    if (kernel) *kernel = plan->kernel;
    return GDN_OK;
}

gdn_status gdn_plan_launches(gdn_plan_t plan, int32_t* launches) {
    if (!plan || !launches) return GDN_ERR_INVALID_ARG;
    *launches = plan->kind == gdn::kFused && !plan->fused_one_launch ? 2 : 1;
    return GDN_OK;
}

size_t gdn_workspace_bytes(gdn_plan_t plan) {
    (void)plan;
    return sizeof(WorkspaceHeader);
}

gdn_status gdn_tail_replay_state(gdn_plan_t plan, const void* q, const void* k, const void* v,
                                 const float* alpha, const float* beta,
                                 const int32_t* seq_offsets, const int32_t* match_len,
                                 const int32_t* R, float* state_out, void* workspace,
                                 void* stream) {
    gdn_status s = check_call_common(plan, workspace);
    if (s != GDN_OK) return s;
    if (plan->kind != gdn::kReplay) return GDN_ERR_INVALID_ARG;
    if (!state_out || !aligned16(state_out)) return GDN_ERR_INVALID_ARG;
    if (plan->total_tokens > 0) {
        if (!k || !v || !alpha || !beta) return GDN_ERR_INVALID_ARG;
        if (!aligned16(k) || !aligned16(v) || !aligned16(alpha) || !aligned16(beta))
            return GDN_ERR_INVALID_ARG;
    }
    CallArgs a;
    std::memset(&a, 0, sizeof a);
    fill_common(plan, a, workspace);
    a.chk_offsets = seq_offsets;
    a.chk_match = match_len;
    a.chk_budget = R;
    a.q = q;
    a.k = k;
    a.v = v;
    a.alpha = alpha;
    a.beta = beta;
    a.state_in = nullptr;
    a.o_out = nullptr;
    a.state_out = state_out;
    return launch(plan, a, static_cast<cudaStream_t>(stream));
}

gdn_status gdn_tail_replay_outputs(gdn_plan_t plan, const void* q, const void* k, const void* v,
                                   const float* alpha, const float* beta,
                                   const int32_t* seq_offsets, const int32_t* match_len,
                                   const int32_t* R, void* o_out, float* state_out, void* workspace,
                                   void* stream) {
    gdn_status s = check_call_common(plan, workspace);
    if (s != GDN_OK) return s;
    if (plan->kind != gdn::kReplay) return GDN_ERR_INVALID_ARG;
    if (state_out && !aligned16(state_out)) return GDN_ERR_INVALID_ARG;
    if (!o_out) return GDN_ERR_INVALID_ARG;   // selects the output-writing kernels
    if (plan->total_tokens > 0) {
        if (!q || !k || !v || !alpha || !beta) return GDN_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(alpha) || !aligned16(beta) ||
            !aligned16(o_out))
            return GDN_ERR_INVALID_ARG;
    }
    CallArgs a;
    std::memset(&a, 0, sizeof a);
    fill_common(plan, a, workspace);
    a.chk_offsets = seq_offsets;
    a.chk_match = match_len;
    a.chk_budget = R;
    a.q = q;
    a.k = k;
    a.v = v;
    a.alpha = alpha;
    a.beta = beta;
    a.state_in = nullptr;
    a.o_out = o_out;
    a.state_out = state_out;
    return launch(plan, a, static_cast<cudaStream_t>(stream));
}

gdn_status gdn_decode_step(int32_t batch, int32_t num_heads, int32_t d_k, int32_t d_v, int32_t dtype,
                           const void* q, const void* k, const void* v, const float* alpha,
                           const float* beta, const float* state_in, float* state_out, void* o_out,
                           void* stream) {
    if (batch < 0 || num_heads < 1) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if ((d_k != 64 && d_k != 128) || (d_v != 64 && d_v != 128)) return GDN_ERR_UNSUPPORTED;
    if ((long long)batch * num_heads > (1ll << 31) - 1) return GDN_ERR_INVALID_ARG;   // grid x
    if (batch == 0) return GDN_OK;
    if (!q || !k || !v || !alpha || !beta || !o_out) return GDN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(alpha) || !aligned16(beta) ||
        !aligned16(o_out) || (state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
        return GDN_ERR_INVALID_ARG;
    gdn::DecodeArgs a;
    std::memset(&a, 0, sizeof a);
    a.dtype = dtype;
    a.num_heads = num_heads;
    a.dk = d_k;
    a.dv = d_v;
    a.batch = batch;
    a.q = q;
    a.k = k;
    a.v = v;
    a.alpha = alpha;
    a.beta = beta;
    a.state_in = state_in;
    a.state_out = state_out;
    a.o_out = o_out;
    if (gdn::launch_decode(a, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_CUDA;
    }
    return GDN_OK;
}

gdn_status gdn_chunk_prefill(gdn_plan_t plan, const void* q, const void* k, const void* v,
                             const float* alpha, const float* beta, const int32_t* cu_seqlens,
                             const float* state_in, void* o_out, float* state_out,
                             void* workspace, void* stream) {
    gdn_status s = check_call_common(plan, workspace);
    if (s != GDN_OK) return s;
    if (plan->kind != gdn::kPrefill) return GDN_ERR_INVALID_ARG;
    if (plan->total_tokens > 0) {
        if (!q || !k || !v || !alpha || !beta || !o_out) return GDN_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(alpha) ||
            !aligned16(beta) || !aligned16(o_out))
            return GDN_ERR_INVALID_ARG;
    }
    if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
        return GDN_ERR_INVALID_ARG;
    CallArgs a;
    std::memset(&a, 0, sizeof a);
    fill_common(plan, a, workspace);
    a.chk_offsets = cu_seqlens;
    a.q = q;
    a.k = k;
    a.v = v;
    a.alpha = alpha;
    a.beta = beta;
    a.state_in = state_in;
    a.o_out = o_out;
    a.state_out = state_out;
    return launch(plan, a, static_cast<cudaStream_t>(stream));
}

gdn_status gdn_tail_replay_prefill(gdn_plan_t plan, const void* k, const void* v, const float* alpha,
                                   const float* beta, const void* sq, const void* sk, const void* sv,
                                   const float* salpha, const float* sbeta, void* o_out, float* state_mid,
                                   float* state_out, void* workspace, void* stream) {
    gdn_status s = check_call_common(plan, workspace);
    if (s != GDN_OK) return s;
    if (plan->kind != gdn::kFused) return GDN_ERR_INVALID_ARG;
    if (!state_out || !aligned16(state_out) || (state_mid && !aligned16(state_mid))) return GDN_ERR_INVALID_ARG;
    long long win_tokens = 0, suf_tokens = 0;
    for (const Window& w : plan->windows0) win_tokens += w.len;
    for (const Window& w : plan->windows) suf_tokens += w.len;
    if (win_tokens > 0) {
        if (!k || !v || !alpha || !beta) return GDN_ERR_INVALID_ARG;
        if (!aligned16(k) || !aligned16(v) || !aligned16(alpha) || !aligned16(beta)) return GDN_ERR_INVALID_ARG;
    }
    if (suf_tokens > 0) {
        if (!sq || !sk || !sv || !salpha || !sbeta || !o_out) return GDN_ERR_INVALID_ARG;
        if (!aligned16(sq) || !aligned16(sk) || !aligned16(sv) || !aligned16(salpha) || !aligned16(sbeta) ||
            !aligned16(o_out))
            return GDN_ERR_INVALID_ARG;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    CallArgs a;
    std::memset(&a, 0, sizeof a);
    fill_common(plan, a, workspace);
    if (plan->fused_one_launch) {
        // one launch: window chunks, then suffix chunks, the state kept on chip
        a.kind = gdn::kFused;
        a.q = sq;
        a.k = sk;
        a.v = sv;
        a.alpha = salpha;
        a.beta = sbeta;
        a.o_out = o_out;
        a.state_out = state_out;
        a.windows0 = plan->d_windows0;
        a.rows_total0 = plan->rows_total0;
        a.k0 = k;
        a.v0 = v;
        a.alpha0 = alpha;
        a.beta0 = beta;
        a.state_mid = state_mid;
        return launch(plan, a, st);
    }
    // two launches under one call number: the state-only replay of the windows into
    // state_mid (or state_out), then the prefill of the suffix from that state
    auto run = plan->kernel == GDN_KERNEL_CHUNKED_TC ? gdn::launch_chunk_tc : gdn::launch_recurrent;
    float* mid = state_mid ? state_mid : state_out;
    a.kind = gdn::kReplay;
    a.windows = plan->d_windows0;
    a.rows_total = plan->rows_total0;
    a.k = k;
    a.v = v;
    a.alpha = alpha;
    a.beta = beta;
    a.state_out = mid;
    if (run(a, st) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_CUDA;
    }
    const unsigned int call = a.epoch;
    fill_common(plan, a, workspace);
    a.epoch = call;
    a.kind = gdn::kPrefill;
    a.q = sq;
    a.k = sk;
    a.v = sv;
    a.alpha = salpha;
    a.beta = sbeta;
    a.state_in = mid;
    a.o_out = o_out;
    a.state_out = state_out;
    if (run(a, st) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_CUDA;
    }
    return GDN_OK;
}

gdn_status gdn_workspace_status(const void* workspace, void* stream) {
    if (!workspace) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_CUDA;
    }
    WorkspaceHeader h;
    if (cudaMemcpy(&h, workspace, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_CUDA;
    }
    const unsigned int status = gdn::header_status(h);
    if (status & gdn::kStatusTimeout) return GDN_ERR_TIMEOUT;
    if (status & gdn::kStatusBounds) return GDN_ERR_BOUNDS;
    if (status & gdn::kStatusMismatch) return GDN_ERR_MISMATCH;
    return GDN_OK;
}

void gdn_debug_fail_plan_allocations(int32_t count) {
    g_fail_plan_allocs.store(count > 0 ? count : 0, std::memory_order_relaxed);
}

const char* gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case GDN_ERR_CUDA: return "CUDA error";
        case GDN_ERR_TIMEOUT: return "device wait timed out";
        case GDN_ERR_ALLOC: return "allocation failed";
        case GDN_ERR_MISMATCH: return "device descriptor arrays disagree with the plan";
        case GDN_ERR_BOUNDS: return "device index outside the plan's extents (debug build)";
    }
    return "unknown status";
}

int32_t gdn_version(void) { return 300; }

}  // extern "C"
