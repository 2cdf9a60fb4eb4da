// gdn_noalloc.cu -- tail replay for callers that cannot allocate device memory.
//
// Some callers run where cudaMalloc is not available to them: code inside a
// memory pool that owns every byte of the device heap, or an allocator-free
// host runtime that only hands out its own input and output buffers.  Such
// callers cannot create a plan (its schedule table is device memory) nor
// provide a workspace.  gdn_tail_replay_state_noalloc() serves them: the
// schedule table and the status word live in one file-scope __device__
// array of fixed size, which every GPU that loads this library holds until
// the process exits.  Nothing here calls cudaMalloc, cudaFree or any
// allocating routine; the host-side schedule is built in a per-thread static
// buffer (not on the stack: the callers this serves may run on threads with
// small stacks).
//
// The array is shared by every call on a device and keeps the last call's
// contents: each call rewrites the schedule and clears the status word
// first, on the caller's stream.  Calls whose work overlaps on the GPU
// (different streams, or several host threads at once) race on it.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "gdn_internal.h"
#include "gdn_tail_replay.h"

namespace {

constexpr size_t kScratchBytes = 64 * 1024;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the scratch array in the current device's context.  It is
// resolved on every call (a cheap host lookup once the module is loaded): a
// cached address would go stale if the context were destroyed and recreated
// (cudaDeviceReset), since the array can then land elsewhere.  The first call
// on a device also loads this library's device code there.
void* scratch_address() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return p;
}

// Host staging of the schedule, one buffer per host thread.  cudaMemcpyAsync
// from pageable memory has read the source by the time it returns, so the
// next call on the same thread may overwrite it at once.
thread_local unsigned char t_host_stage[kScratchBytes] __attribute__((aligned(16)));

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" gdn_status gdn_tail_replay_state_noalloc(const gdn_varlen_desc* cache,
                                                   const int32_t* match_len_host,
                                                   const int32_t* R_host, const void* k,
                                                   const void* v, const float* alpha,
                                                   const float* beta, float* state_out,
                                                   void* stream, uint32_t* status_out) {
    using gdn::CallArgs;
    using gdn::Unit;
    using gdn::Window;
    using gdn::WorkspaceHeader;
    // the same descriptor checks a replay plan makes
    gdn_status s0 = gdn::check_varlen_desc(cache);
    if (s0 != GDN_OK) return s0;
    if (!match_len_host || !R_host) return GDN_ERR_INVALID_ARG;
    const int batch = cache->batch, H = cache->num_heads;
    const size_t need = sizeof(WorkspaceHeader) + sizeof(Window) * (size_t)batch +
                        sizeof(Unit) * (size_t)batch * (size_t)H;
    if (need > kScratchBytes) return GDN_ERR_UNSUPPORTED;   // beyond the fixed scratch
    int kernel = gdn::kernel_family_of(cache->kernel);
    const bool tc_ok = gdn::chunk_tc_supported(cache->dtype, cache->d_k, cache->d_v);
    if (kernel == GDN_KERNEL_AUTO) kernel = tc_ok ? GDN_KERNEL_CHUNKED_TC : GDN_KERNEL_RECURRENT;
    if (kernel == GDN_KERNEL_CHUNKED_TC && !tc_ok) return GDN_ERR_UNSUPPORTED;

    // Host staging of the schedule: windows, then units longest window first.
    // Temporaries (window rows and lengths, sequence order) sit after it.
    const size_t tmp_bytes = (sizeof(int64_t) + 2 * sizeof(int32_t)) * (size_t)batch;
    if (need + tmp_bytes > kScratchBytes) return GDN_ERR_UNSUPPORTED;
    unsigned char* host = t_host_stage;
    Window* win = reinterpret_cast<Window*>(host + sizeof(WorkspaceHeader));
    Unit* units = reinterpret_cast<Unit*>(host + sizeof(WorkspaceHeader) + sizeof(Window) * batch);
    int64_t* row0 = reinterpret_cast<int64_t*>(host + ((need + 15) & ~size_t(15)));
    int32_t* len = reinterpret_cast<int32_t*>(row0 + batch);
    int32_t* order = len + batch;
    if (reinterpret_cast<unsigned char*>(order + batch) > host + kScratchBytes) return GDN_ERR_UNSUPPORTED;
    {
        // the same windows a replay plan would use, without its allocations
        gdn_status s = gdn_replay_windows(batch, cache->seq_offsets_host, match_len_host, R_host, row0, len);
        if (s != GDN_OK) return s;
        const int32_t* off = cache->seq_offsets_host;
        long long total = 0, rows_total = 0;
        for (int b = 0; b < batch; ++b) {
            Window w;
            std::memset(&w, 0, sizeof w);
            w.row0 = row0[b];
            w.len = len[b];
            w.expect_off = off[b];
            w.expect_end = off[b + 1];
            w.expect_match = match_len_host[b];
            w.expect_budget = R_host[b];
            win[b] = w;
            total += w.len;
            if (off[b + 1] > rows_total) rows_total = off[b + 1];
        }
        // sequences by window length, longest first (stable insertion sort)
        for (int b = 0; b < batch; ++b) {
            int j = b;
            while (j > 0 && win[order[j - 1]].len < win[b].len) {
                order[j] = order[j - 1];
                --j;
            }
            order[j] = b;
        }
        for (int i = 0; i < batch; ++i)
            for (int h = 0; h < H; ++h) units[(size_t)i * H + h] = Unit{order[i], h};

        if (total > 0) {
            if (!k || !v || !alpha || !beta) return GDN_ERR_INVALID_ARG;
            if (!aligned16(k) || !aligned16(v) || !aligned16(alpha) || !aligned16(beta))
                return GDN_ERR_INVALID_ARG;
        }
        if (!state_out || !aligned16(state_out)) return GDN_ERR_INVALID_ARG;

        unsigned char* scratch = static_cast<unsigned char*>(scratch_address());
        if (!scratch) return GDN_ERR_CUDA;
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        std::memset(host, 0, sizeof(WorkspaceHeader));   // no status reported under any call number
        if (cudaMemcpyAsync(scratch, host, need, cudaMemcpyHostToDevice, st) != cudaSuccess) {
            cudaGetLastError();
            return GDN_ERR_CUDA;
        }
        CallArgs a;
        std::memset(&a, 0, sizeof a);
        a.kind = gdn::kReplay;
        a.dtype = cache->dtype;
        a.num_heads = H;
        a.dk = cache->d_k;
        a.dv = cache->d_v;
        a.batch = batch;
        a.units = (long long)batch * H;
        a.rows_total = rows_total;
        a.rs_qk = gdn::row_stride_qk(cache);
        a.rs_v = gdn::row_stride_v(cache);
        a.windows = reinterpret_cast<const Window*>(scratch + sizeof(WorkspaceHeader));
        a.unit_list = reinterpret_cast<const Unit*>(scratch + sizeof(WorkspaceHeader) + sizeof(Window) * batch);
        a.k = k;
        a.v = v;
        a.alpha = alpha;
        a.beta = beta;
        a.state_out = state_out;
        a.ws = reinterpret_cast<WorkspaceHeader*>(scratch);
        a.epoch = gdn::next_call_number();
        a.replay_variant = gdn::replay_variant_of(cache->kernel);
        cudaError_t e = kernel == GDN_KERNEL_CHUNKED_TC ? gdn::launch_chunk_tc(a, st) : gdn::launch_recurrent(a, st);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return GDN_ERR_CUDA;
        }
        if (status_out) {
            WorkspaceHeader hdr;
            if (cudaMemcpyAsync(&hdr, scratch, sizeof hdr, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
                cudaStreamSynchronize(st) != cudaSuccess) {
                cudaGetLastError();
                return GDN_ERR_CUDA;
            }
            *status_out = gdn::header_status(hdr);
        }
    }
    return GDN_OK;
}
