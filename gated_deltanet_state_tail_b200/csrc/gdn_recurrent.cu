// gdn_recurrent.cu -- exact fp32 token-recurrent kernel for the gated delta rule.
//
// One CTA per (sequence, head, 64-column block).  Column c of the d_k x d_v state lives in
// the registers of d_k / 64 adjacent lanes (64 key rows each), so k_t^T S (a
// per-column dot product over the key dimension) needs at most one shuffle
// and the rank-1 update is thread-local.
//
// The rule (Gated DeltaNet, the recurrence that Tail-Replay replays; "Tail-Replay:
// Escaping the Curse of Linear Attention in Prefix Caching for Hybrid LLMs",
// section "Mecanismos Principais", item "Reconstrucao de Estado Independente"):
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
// is rewritten per column as S_t = alpha_t S_{t-1} + k_t u_t^T with
//   u_t = beta_t (v_t - alpha_t S_{t-1}^T k_t).
// The decay is carried as a scalar: S = sigma * Stilde, so a token costs two
// FMAs per state element (dot product and update) instead of three; sigma is
// folded back into Stilde when it gets small (or the gate is exactly 0).
//
// This kernel is the fp32 path (1e-4 tolerance) and serves any supported
// shape; the tensor-core chunked kernel serves bf16 with d = 128.
#include <cuda_bf16.h>

#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kStageTokens = 16;  // 24 KB of fp32 staging at d = 128 with outputs
constexpr float kRenormBelow = 1e-20f;

template <typename T>
__device__ __forceinline__ void load4(const T* src, float* dst);

template <>
__device__ __forceinline__ void load4<float>(const float* src, float* dst) {
    float4 x = *reinterpret_cast<const float4*>(src);
    dst[0] = x.x; dst[1] = x.y; dst[2] = x.z; dst[3] = x.w;
}

template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* src, float* dst) {
    uint2 x = *reinterpret_cast<const uint2*>(src);
    dst[0] = __uint_as_float(x.x << 16);
    dst[1] = __uint_as_float(x.x & 0xffff0000u);
    dst[2] = __uint_as_float(x.y << 16);
    dst[3] = __uint_as_float(x.y & 0xffff0000u);
}

__device__ __forceinline__ void store1(float* p, float x) { *p = x; }
__device__ __forceinline__ void store1(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Stage rows [t0, t0 + n) of one head (n <= kStageTokens) into shared memory
// as fp32.  Element loads are 4-wide vectors: every row stride is a multiple
// of 16 bytes (the host checks it) and d_k, d_v are multiples of 64.
template <typename T, int DK, int DV, bool OUT>
__device__ __forceinline__ void stage_rows(const CallArgs& a, long long row0, int t0, int n, int h,
                                           float* sk, float* sv, float* sq, float* sa, float* sb) {
    const int H = a.num_heads;
    const T* k = static_cast<const T*>(a.k);
    const T* v = static_cast<const T*>(a.v);
    const T* q = static_cast<const T*>(a.q);
    for (int e = threadIdx.x * 4; e < n * DK; e += blockDim.x * 4) {
        int j = e / DK, i = e % DK;
        if (!index_ok(a, row0 + t0 + j < a.rows_total)) continue;
        long long g = (row0 + t0 + j) * a.rs_qk + (long long)h * DK + i;
        load4<T>(k + g, sk + e);
        if (OUT) load4<T>(q + g, sq + e);
    }
    for (int e = threadIdx.x * 4; e < n * DV; e += blockDim.x * 4) {
        int j = e / DV, i = e % DV;
        if (!index_ok(a, row0 + t0 + j < a.rows_total)) continue;
        long long g = (row0 + t0 + j) * a.rs_v + (long long)h * DV + i;
        load4<T>(v + g, sv + e);
    }
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        if (!index_ok(a, row0 + t0 + j < a.rows_total)) continue;
        long long g = (row0 + t0 + j) * H + h;
        sa[j] = a.alpha[g];
        sb[j] = a.beta[g];
    }
}

// Thread layout: KS = DK / 64 threads share one state column (lanes 2c and
// 2c+1 when DK = 128); each holds 64 consecutive key rows of the column and
// the partial dot products are combined with one shuffle.
template <typename T, int DK, int DV, bool OUT>
__global__ void __launch_bounds__(64 * (DK / 64), 3) recurrent_kernel(const CallArgs a) {
    constexpr int KS = DK / 64;        // threads per column
    constexpr int KR = 64;             // key rows per thread
    constexpr int COLS = 64;           // state columns per CTA; blockIdx.y picks the block
    __shared__ __align__(16) float sk[kStageTokens * DK];
    __shared__ __align__(16) float sq[OUT ? kStageTokens * DK : 4];
    __shared__ __align__(16) float sv[kStageTokens * DV];
    __shared__ float sa[kStageTokens], sb[kStageTokens];

    record_call(a);
    const Unit u = a.unit_list[blockIdx.x];
    const int b = u.seq, h = u.head;
    const int c = blockIdx.y * COLS + threadIdx.x / KS, part = threadIdx.x % KS, r0 = part * KR;
    if (!window_agrees(a, b)) {
        if (threadIdx.x == 0) report_status(a, kStatusMismatch);
        return;
    }
    const Window w = a.windows[b];
    const size_t state_base = ((size_t)b * a.num_heads + h) * DK * DV;
    // debug build: the unit, its column block and its window lie inside the plan (uniform)
    if (!index_ok(a, b >= 0 && b < a.batch && h >= 0 && h < a.num_heads && blockIdx.y * COLS + COLS <= DV &&
                            w.row0 >= 0 && w.len >= 0 && w.row0 + w.len <= a.rows_total))
        return;

    float s[KR];
    float sigma = 1.0f;
    if (a.state_in) {
#pragma unroll
        for (int i = 0; i < KR; ++i) s[i] = a.state_in[state_base + (size_t)(r0 + i) * DV + c];
    } else {
#pragma unroll
        for (int i = 0; i < KR; ++i) s[i] = 0.0f;
    }

    T* o = static_cast<T*>(a.o_out);
    for (int t0 = 0; t0 < w.len; t0 += kStageTokens) {
        const int n = min(kStageTokens, w.len - t0);
        __syncthreads();
        stage_rows<T, DK, DV, OUT>(a, w.row0, t0, n, h, sk, sv, sq, sa, sb);
        __syncthreads();
        for (int j = 0; j < n; ++j) {
            const float* kt = sk + j * DK + r0;
            const float al = sa[j], be = sb[j];
            // dot = (S_{t-1}^T k_t)_c = sigma * sum_i k_i Stilde_i
            float p[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) p[m] = 0.0f;
#pragma unroll
            for (int i = 0; i < KR; i += 4) {
                float4 kk = *reinterpret_cast<const float4*>(kt + i);
                float& acc = p[(i / 4) % 8];
                acc = fmaf(kk.x, s[i], acc);
                acc = fmaf(kk.y, s[i + 1], acc);
                acc = fmaf(kk.z, s[i + 2], acc);
                acc = fmaf(kk.w, s[i + 3], acc);
            }
            float dot = ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
            if (KS == 2) dot += __shfl_xor_sync(0xffffffffu, dot, 1);
            dot *= sigma;
            const float uc = be * (sv[j * DV + c] - al * dot);
            // S_t = alpha S_{t-1} + k u^T, with S = sigma * Stilde
            float ns = al * sigma;
            float coef;
            if (ns < kRenormBelow) {      // uniform across the CTA: al, sigma are per unit
#pragma unroll
                for (int i = 0; i < KR; ++i) s[i] *= ns;
                ns = 1.0f;
                coef = uc;
            } else {
                coef = uc / ns;
            }
            sigma = ns;
#pragma unroll
            for (int i = 0; i < KR; i += 4) {
                float4 kk = *reinterpret_cast<const float4*>(kt + i);
                s[i] = fmaf(kk.x, coef, s[i]);
                s[i + 1] = fmaf(kk.y, coef, s[i + 1]);
                s[i + 2] = fmaf(kk.z, coef, s[i + 2]);
                s[i + 3] = fmaf(kk.w, coef, s[i + 3]);
            }
            if (OUT) {
                // o_t = S_t^T q_t
                const float* qt = sq + j * DK + r0;
#pragma unroll
                for (int m = 0; m < 8; ++m) p[m] = 0.0f;
#pragma unroll
                for (int i = 0; i < KR; i += 4) {
                    float4 qq = *reinterpret_cast<const float4*>(qt + i);
                    float& acc = p[(i / 4) % 8];
                    acc = fmaf(qq.x, s[i], acc);
                    acc = fmaf(qq.y, s[i + 1], acc);
                    acc = fmaf(qq.z, s[i + 2], acc);
                    acc = fmaf(qq.w, s[i + 3], acc);
                }
                float ov = ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
                if (KS == 2) ov += __shfl_xor_sync(0xffffffffu, ov, 1);
                if (part == 0 && index_ok(a, w.row0 + t0 + j < a.rows_total))
                    store1(o + ((w.row0 + t0 + j) * a.num_heads + h) * (long long)DV + c, sigma * ov);
            }
        }
    }
    if (a.state_out) {
#pragma unroll
        for (int i = 0; i < KR; ++i) a.state_out[state_base + (size_t)(r0 + i) * DV + c] = sigma * s[i];
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_typed(const CallArgs& a, cudaStream_t stream) {
    dim3 grid((unsigned)a.units, DV / 64), block(64 * (DK / 64));
    if (a.kind == kPrefill || a.o_out)   // outputs: a prefill, or a replay that emits them
        recurrent_kernel<T, DK, DV, true><<<grid, block, 0, stream>>>(a);
    else
        recurrent_kernel<T, DK, DV, false><<<grid, block, 0, stream>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dims(const CallArgs& a, cudaStream_t stream) {
    if (a.dk == 64 && a.dv == 64) return launch_typed<T, 64, 64>(a, stream);
    if (a.dk == 64 && a.dv == 128) return launch_typed<T, 64, 128>(a, stream);
    if (a.dk == 128 && a.dv == 64) return launch_typed<T, 128, 64>(a, stream);
    if (a.dk == 128 && a.dv == 128) return launch_typed<T, 128, 128>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_recurrent(const CallArgs& a, cudaStream_t stream) {
    if (a.units == 0) return cudaSuccess;
    if (a.dtype == 0) return launch_dims<float>(a, stream);
    return launch_dims<__nv_bfloat16>(a, stream);
}

}  // namespace gdn
