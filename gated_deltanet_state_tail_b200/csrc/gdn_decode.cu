// gdn_decode.cu -- one decode step of the gated delta rule: the token that
// follows the suffix prefill (the first generated token whose latency the
// Tail-Replay pages time as TTFT; "Tail-Replay: Escaping the Curse of Linear
// Attention in Prefix Caching for Hybrid LLMs", section "Resultados").
//
// Per (request, head), with the d_k x d_v state S (rows = key index):
//   S' = alpha (I - beta k k^T) S + beta k v^T = alpha S + k u^T,
//   u  = beta (v - alpha S^T k),          o = S'^T q.
// The step reads and writes the whole state once and does 6 d_k d_v flops on
// it, so it is bound by HBM (2 d_k d_v 4 bytes per head).
//
// Layout of the work: one CTA of 256 threads per (request, head, block of 32
// value columns).  Lane l owns column 32 blockIdx.y + l, so each state row a
// warp touches is one coalesced 128-byte line; warp w owns key rows
// [w d_k / 8, (w + 1) d_k / 8) in registers.  The two per-column dot products
// (S^T k and S'^T q) are summed over the eight warps through shared memory.
// Each state element is read and written by the same thread, so the update
// may run in place (state_out == state_in).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCols = 32;   // value columns per CTA

__device__ __forceinline__ float load_elt(const float* p) { return *p; }
__device__ __forceinline__ float load_elt(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void store_elt(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_elt(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeArgs a) {
    constexpr int RW = DK / kWarps;   // key rows per thread
    __shared__ float sk[DK], sq[DK];
    __shared__ float red[kWarps][kCols];

    const int bh = blockIdx.x;                  // request * H + head
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.y * kCols + lane;    // value column of this thread
    const int r0 = warp * RW;                   // first key row of this thread
    const T* q = static_cast<const T*>(a.q) + (size_t)bh * DK;
    const T* k = static_cast<const T*>(a.k) + (size_t)bh * DK;
    for (int i = tid; i < DK; i += kThreads) {
        sk[i] = load_elt(k + i);
        sq[i] = load_elt(q + i);
    }
    const float al = a.alpha[bh], be = a.beta[bh];
    const float vc = load_elt(static_cast<const T*>(a.v) + (size_t)bh * DV + c);
    const size_t base = (size_t)bh * DK * DV + c;

    float s[RW];
    if (a.state_in) {
#pragma unroll
        for (int r = 0; r < RW; ++r) s[r] = a.state_in[base + (size_t)(r0 + r) * DV];
    } else {
#pragma unroll
        for (int r = 0; r < RW; ++r) s[r] = 0.0f;
    }
    __syncthreads();

    // (S^T k)_c
    float d0 = 0.0f, d1 = 0.0f;
#pragma unroll
    for (int r = 0; r < RW; r += 2) {
        d0 = fmaf(s[r], sk[r0 + r], d0);
        d1 = fmaf(s[r + 1], sk[r0 + r + 1], d1);
    }
    red[warp][lane] = d0 + d1;
    __syncthreads();
    float dot = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) dot += red[w][lane];
    const float u = be * (vc - al * dot);

    // S' = alpha S + k u^T, then (S'^T q)_c
    float o0 = 0.0f, o1 = 0.0f;
#pragma unroll
    for (int r = 0; r < RW; ++r) {
        s[r] = fmaf(sk[r0 + r], u, al * s[r]);
        if (r & 1) o1 = fmaf(s[r], sq[r0 + r], o1);
        else o0 = fmaf(s[r], sq[r0 + r], o0);
    }
    __syncthreads();   // every thread has read red[] for the first sum
    red[warp][lane] = o0 + o1;
    if (a.state_out) {
#pragma unroll
        for (int r = 0; r < RW; ++r) a.state_out[base + (size_t)(r0 + r) * DV] = s[r];
    }
    __syncthreads();
    if (warp == 0) {
        float ov = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) ov += red[w][lane];
        store_elt(static_cast<T*>(a.o_out) + (size_t)bh * DV + c, ov);
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_typed(const DecodeArgs& a, cudaStream_t stream) {
    const dim3 grid((unsigned)((long long)a.batch * a.num_heads), DV / kCols);
    decode_kernel<T, DK, DV><<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dims(const DecodeArgs& a, cudaStream_t stream) {
    if (a.dk == 64 && a.dv == 64) return launch_typed<T, 64, 64>(a, stream);
    if (a.dk == 64 && a.dv == 128) return launch_typed<T, 64, 128>(a, stream);
    if (a.dk == 128 && a.dv == 64) return launch_typed<T, 128, 64>(a, stream);
    if (a.dk == 128 && a.dv == 128) return launch_typed<T, 128, 128>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    if (a.batch == 0) return cudaSuccess;
    if (a.dtype == 0) return launch_dims<float>(a, stream);
    return launch_dims<__nv_bfloat16>(a, stream);
}

}  // namespace gdn
