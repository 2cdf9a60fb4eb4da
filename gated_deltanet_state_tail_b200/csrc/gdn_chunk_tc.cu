// gdn_chunk_tc.cu -- chunked gated-delta-rule kernel on tcgen05 tensor cores
// (bf16 q/k/v, d_k = d_v = 128, fp32 state in tensor memory).
//
// The recurrence (Gated DeltaNet, replayed by Tail-Replay: "Tail-Replay:
// Escaping the Curse of Linear Attention in Prefix Caching for Hybrid LLMs",
// section "Mecanismos Principais", item "Reconstrucao de Estado
// Independente"):  S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
// o_t = S_t^T q_t, is evaluated 64 tokens at a time in the chunkwise (WY / UT)
// form of the delta rule (Yang et al., "Parallelizing Linear Transformers with
// the Delta Rule over Sequence Length", 2024, with the gate folded in).  With
// S0 the state entering a chunk, gamma_i = prod_{m<=i} alpha_m and
// G_i = log gamma_i:
//   A_ij = beta_i exp(G_i - G_j) k_i.k_j  (i > j),   T = (I + A)^-1
//   W    = T diag(beta gamma) K,   U' = T diag(beta) V           (S-independent)
//   U    = U' - W S0
//   S_C  = gamma_C S0 + K^T diag(gamma_C / gamma) U
//   O    = diag(gamma) Q S0 + (tril(Q K^T) * exp(G_i - G_j)) U
// Every contraction is a tcgen05.mma with M = 128 (the key or value
// dimension, or the 64 chunk rows of K stacked on 64 rows of Q/V), operands in
// 128-byte-swizzled shared memory (TMA-loaded tiles or tiles the epilogues
// write), accumulators in TMEM.  T is built on CUDA cores in fp32.
//
// Work: one CTA per (sequence, head) unit, 4 warps, chunks in order.  Thread
// t owns TMEM lane t in every epilogue.  Replay: 96 KB shared memory and 256
// TMEM columns, so two CTAs share an SM and overlap each other's serial
// chain.  Prefill adds the output path (152 KB, 512 columns).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn_internal.h"
#include "gdn_sm100.h"

namespace gdn {
namespace {

using namespace sm100;

constexpr int C = 64;        // chunk length
constexpr int D = 128;       // d_k = d_v
constexpr int NT = 128;      // threads per CTA
constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s per wait
constexpr float kLog2Floor = -115.0f;         // log2 of a zero gate, clamped (2^-115 ~ 2.4e-35)

// ---- shared memory map (byte offsets from a 1 KB aligned base) ----
// TILE: [K0 | X0 | K1 | X1], 8 KB boxes of 64 rows x 64 columns.  X = V
//       (replay) or Q (prefill).  Block kb holds columns [64 kb, 64 kb + 64).
// VT  : prefill only, [V0 | V1].
// SB  : bf16 S as an MN-major operand (two 16 KB dv-blocks of 128 k-rows);
//       during the chunk prep it holds A (fp32 64 x 64) and scratch.
// UT  : bf16 diag(gamma_C / gamma) U, [dv][j]; during prep T diag(beta) and
//       T diag(beta gamma) in bf16.
// WT  : bf16 -W^T, [dk][j]; during prep T in fp32.
// UB  : prefill, bf16 U^T unscaled, [dv][j].
// MB  : prefill, bf16 masked decayed Q K^T, [i][j].
// GQ  : prefill, bf16 diag(gamma) Q, [i][dk] as two 8 KB blocks.
constexpr uint32_t OFF_TILE = 0;
constexpr uint32_t OFF_SB = 32768;
constexpr uint32_t OFF_UT = OFF_SB + 32768;
constexpr uint32_t OFF_WT = OFF_UT + 16384;
constexpr uint32_t SMEM_REPLAY = OFF_WT + 16384;        // 96 KB
constexpr uint32_t OFF_VT = SMEM_REPLAY;
constexpr uint32_t OFF_UB = OFF_VT + 16384;
constexpr uint32_t OFF_MB = OFF_UB + 16384;
constexpr uint32_t OFF_GQ = OFF_MB + 8192;
constexpr uint32_t SMEM_PREFILL = OFF_GQ + 16384;       // 152 KB
// fp32 scratch inside SB during the prep
constexpr uint32_t OFF_A = OFF_SB;                      // 64 x 64 fp32
constexpr uint32_t OFF_P = OFF_SB + 16384;              // up to 3 x 256 fp32
constexpr uint32_t OFF_T = OFF_WT;                      // 64 x 64 fp32
constexpr uint32_t OFF_TB = OFF_UT;                     // bf16 T diag(beta)
constexpr uint32_t OFF_TBG = OFF_UT + 8192;             // bf16 T diag(beta gamma)

// TMEM columns
constexpr uint32_t TM_S = 0;      // 128 columns: fp32 S, lane = key row
constexpr uint32_t TM_U = 128;    // 64 columns: U'^T then U^T, lane = value row
constexpr uint32_t TM_P = 192;    // 64 columns: [K;X] K^T, then W^T
constexpr uint32_t TM_O = 256;    // 64 columns (prefill): O^T

struct TcParams {
    CallArgs a;
    long long rows_total;
};

__device__ __forceinline__ void st_shared_v4(uint8_t* base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4*>(base + off) = v;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

// Write 64 fp32 values (one row, columns 0..63) as bf16 into a 128-byte
// swizzled row `row` of the tile at `tile`.
__device__ __forceinline__ void write_row64_bf16(uint8_t* tile, int row, const float* v) {
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        uint4 q;
        q.x = pack_bf16(v[ch * 8 + 0], v[ch * 8 + 1]);
        q.y = pack_bf16(v[ch * 8 + 2], v[ch * 8 + 3]);
        q.z = pack_bf16(v[ch * 8 + 4], v[ch * 8 + 5]);
        q.w = pack_bf16(v[ch * 8 + 6], v[ch * 8 + 7]);
        st_shared_v4(tile, (uint32_t)(row * 128 + ((ch ^ (row & 7)) << 4)), q);
    }
}

__device__ __forceinline__ float bf16_at(const uint8_t* tile, int row, int col) {
    const __nv_bfloat16 x = *reinterpret_cast<const __nv_bfloat16*>(tile + sw128_offset(row, col));
    return __bfloat162float(x);
}

// Block-wide agreement after a bounded wait: every thread leaves together.
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, const CallArgs& a, uint32_t where) {
    bool ok = mbar_wait_bounded(bar, parity, kWaitNs);
    ok = __syncthreads_and(ok) != 0;
    if (!ok && threadIdx.x == 0) {
        atomicOr(&a.ws->status, kStatusTimeout);
        atomicCAS(&a.ws->timeout_where, 0u, where);
    }
    return ok;
}

// T = (I + A)^-1 for the strictly lower triangular 64 x 64 A (fp32, row
// stride 64), by 16 x 16 diagonal blocks (forward substitution) and the
// block recurrence T_ba = -T_bb sum_{a <= m < b} A_bm T_ma.  Writes T (fp32,
// lower triangle, zeros above) to Ts.
__device__ void invert_unit_lower(const float* As, float* Ts, float* Ps) {
    const int tid = threadIdx.x;
    // zero T
    for (int e = tid; e < C * C; e += NT) Ts[e] = 0.0f;
    __syncthreads();
    if (tid < 64) {
        const int bb = tid >> 4, cc = tid & 15, o = bb * 16;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc = (i == cc) ? 1.0f : 0.0f;
#pragma unroll
            for (int j = 0; j < i; ++j) acc = fmaf(-As[(o + i) * C + o + j], x[j], acc);
            x[i] = (i < cc) ? 0.0f : acc;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Ts[(o + i) * C + o + cc] = x[i];
    }
    __syncthreads();
    for (int b = 1; b < 4; ++b) {
        // P_ba = sum_{m=a}^{b-1} A_bm T_ma for a < b: b * 256 elements
        for (int e = tid; e < b * 256; e += NT) {
            const int a = e >> 8, r = (e >> 4) & 15, cc = e & 15;
            float acc = 0.0f;
            for (int m = a; m < b; ++m) {
#pragma unroll
                for (int l = 0; l < 16; ++l)
                    acc = fmaf(As[(16 * b + r) * C + 16 * m + l], Ts[(16 * m + l) * C + 16 * a + cc], acc);
            }
            Ps[e] = acc;
        }
        __syncthreads();
        for (int e = tid; e < b * 256; e += NT) {
            const int a = e >> 8, r = (e >> 4) & 15, cc = e & 15;
            float acc = 0.0f;
#pragma unroll
            for (int l = 0; l < 16; ++l)
                acc = fmaf(Ts[(16 * b + r) * C + 16 * b + l], Ps[(a << 8) + (l << 4) + cc], acc);
            Ts[(16 * b + r) * C + 16 * a + cc] = -acc;
        }
        __syncthreads();
    }
}

template <bool REPLAY>
__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(const TcParams p, const __grid_constant__ CUtensorMap map_k,
                const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_q) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar_tma, bar_mma;
    __shared__ uint32_t tmem_slot;
    __shared__ float s_beta[C], s_g2[C], s_gam[C];
    __shared__ float s_scan;

    const CallArgs& a = p.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr uint32_t kTmemCols = REPLAY ? 256 : 512;
    const Unit u = a.unit_list[blockIdx.x];
    const int b = u.seq, h = u.head, H = a.num_heads;

    if (!window_agrees(a, b)) {
        if (tid == 0) atomicOr(&a.ws->status, kStatusMismatch);
        return;
    }
    const Window w = a.windows[b];

    if (tid == 0) {
        mbar_init(&bar_tma, 1);
        mbar_init(&bar_mma, 1);
        mbar_fence_init();
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
        if (!REPLAY) tma_prefetch_desc(&map_q);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_slot;
    const uint32_t tlane = tbase + ((uint32_t)(warp * 32) << 16);   // this thread's lane, column 0

    uint8_t* tile = sm + OFF_TILE;
    uint8_t* vtile = REPLAY ? sm + OFF_TILE + 8192 : sm + OFF_VT;
    const uint32_t v_lbo = REPLAY ? 16384u : 8192u;
    const uint32_t s_tile = smem_u32(tile), s_vtile = smem_u32(vtile);
    const uint32_t s_sb = smem_u32(sm + OFF_SB), s_ut = smem_u32(sm + OFF_UT), s_wt = smem_u32(sm + OFF_WT);
    const uint32_t s_tb = smem_u32(sm + OFF_TB), s_tbg = smem_u32(sm + OFF_TBG);
    const uint32_t s_ub = smem_u32(sm + OFF_UB), s_mb = smem_u32(sm + OFF_MB), s_gq = smem_u32(sm + OFF_GQ);

    // ---- initial state into TMEM (thread t = key row t) ----
    const size_t state_base = ((size_t)b * H + h) * D * D;
    {
        float v[32];
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            if (!REPLAY && a.state_in) {
                const float4* src = reinterpret_cast<const float4*>(a.state_in + state_base + (size_t)tid * D + cb * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float4 x = src[i];
                    v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.0f;
            }
            tmem_st32(tlane + TM_S + cb * 32, v);
        }
        tmem_wait_st();
    }

    const uint32_t id_kk = idesc_bf16(128, 64, false, false);    // [K;X] K^T
    const uint32_t id_w = idesc_bf16(128, 64, true, false);      // K^T (T..)^T, V^T (T..)^T
    const uint32_t id_u = idesc_bf16(128, 64, true, true);       // S^T (-W^T)
    const uint32_t id_o1 = idesc_bf16(128, 64, true, false);     // S^T (gamma Q)^T
    const uint32_t id_s = idesc_bf16(128, 128, true, false);     // K^T U~
    const uint32_t id_o2 = idesc_bf16(128, 64, false, false);    // U^T M^T

    uint32_t ph_tma = 0, ph_mma = 0;
    bool ok = true;
    const int nchunks = (w.len + C - 1) / C;
    const uint32_t tile_bytes = REPLAY ? 4u * 8192u : 6u * 8192u;

    for (int c = 0; c < nchunks && ok; ++c) {
        const long long r0 = w.row0 + (long long)c * C;
        const int nc = min(C, w.len - c * C);

        // ---- load the chunk's tiles (TMA) and gates ----
        if (tid == 0) {
            mbar_arrive_expect_tx(&bar_tma, tile_bytes);
            tma_load_3d(tile, &map_k, &bar_tma, 0, h, (int)r0);
            tma_load_3d(tile + 16384, &map_k, &bar_tma, 64, h, (int)r0);
            tma_load_3d(vtile, &map_v, &bar_tma, 0, h, (int)r0);
            tma_load_3d(vtile + v_lbo, &map_v, &bar_tma, 64, h, (int)r0);
            if (!REPLAY) {
                tma_load_3d(tile + 8192, &map_q, &bar_tma, 0, h, (int)r0);
                tma_load_3d(tile + 24576, &map_q, &bar_tma, 64, h, (int)r0);
            }
        }
        if (tid < C) {
            float al = 1.0f, be = 0.0f;
            if (tid < nc) {
                al = a.alpha[(r0 + tid) * H + h];
                be = a.beta[(r0 + tid) * H + h];
            }
            float lg = al > 0.0f ? fmaxf(__log2f(al), kLog2Floor) : kLog2Floor;
            // inclusive scan over the 64 tokens (two warps)
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                float y = __shfl_up_sync(0xffffffffu, lg, off);
                if (lane >= off) lg += y;
            }
            if (tid == 31) s_scan = lg;
            s_beta[tid] = be;
            s_g2[tid] = lg;   // warp 1 adds warp 0's total below
        }
        __syncthreads();
        if (tid >= 32 && tid < C) s_g2[tid] += s_scan;
        __syncthreads();
        if (tid < C) s_gam[tid] = exp2f(s_g2[tid]);
        ok = wait_all(&bar_tma, ph_tma, a, 1);
        ph_tma ^= 1;
        if (!ok) break;
        if (nc < C) {   // padded tokens are identity transitions: zero their rows
            const int nrows = C - nc;
            const int ntiles = REPLAY ? 4 : 6;
            for (int e = tid; e < ntiles * nrows * 8; e += NT) {
                const int t = e / (nrows * 8), rr = nc + (e / 8) % nrows, ch = e % 8;
                uint8_t* base = (t < 4) ? tile + t * 8192 : vtile + (t - 4) * 8192;
                st_shared_v4(base, (uint32_t)(rr * 128 + ch * 16), make_uint4(0, 0, 0, 0));
            }
            fence_proxy_async_smem();
        }
        __syncthreads();

        // ---- MMA 1: [K; X] K^T -> TM_P (rows 0..63: K K^T, rows 64..127: Q K^T) ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16_ss(tbase + TM_P, smem_desc_sw128(s_tile + off, 16, 1024),
                            smem_desc_sw128(s_tile + off, 16, 1024), id_kk, kk > 0);
            }
            mma_commit(&bar_mma);
        }
        ok = wait_all(&bar_mma, ph_mma, a, 2);
        ph_mma ^= 1;
        if (!ok) break;
        tc_fence_after();

        // ---- epilogue 1: A (rows 0..63) and M (rows 64..127, prefill) ----
        {
            float* As = reinterpret_cast<float*>(sm + OFF_A);
            const bool krow = tid < C;
            if (krow || !REPLAY) {
                const int i = krow ? tid : tid - C;
                const float gi = s_g2[i];
                const float bi = s_beta[i];
                float v[64];
                tmem_ld32(tlane + TM_P, v);
                tmem_ld32(tlane + TM_P + 32, v + 32);
                tmem_wait_ld();
                if (krow) {
#pragma unroll
                    for (int j = 0; j < C; ++j)
                        As[i * C + j] = (j < i) ? bi * exp2f(gi - s_g2[j]) * v[j] : 0.0f;
                } else {
#pragma unroll
                    for (int j = 0; j < C; ++j) v[j] = (j <= i) ? exp2f(gi - s_g2[j]) * v[j] : 0.0f;
                    write_row64_bf16(sm + OFF_MB, i, v);
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- T = (I + A)^-1 and its two scaled bf16 copies ----
        {
            const float* As = reinterpret_cast<const float*>(sm + OFF_A);
            float* Ts = reinterpret_cast<float*>(sm + OFF_T);
            float* Ps = reinterpret_cast<float*>(sm + OFF_P);
            invert_unit_lower(As, Ts, Ps);
            const int j = tid >> 1, half = tid & 1;
            float vb[32], vbg[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const int jp = half * 32 + q;
                const float t = Ts[j * C + jp] * s_beta[jp];
                vb[q] = t;
                vbg[q] = t * s_gam[jp];
            }
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const int chunk = half * 4 + ch;
                uint4 x, y;
                x.x = pack_bf16(vb[ch * 8 + 0], vb[ch * 8 + 1]);
                x.y = pack_bf16(vb[ch * 8 + 2], vb[ch * 8 + 3]);
                x.z = pack_bf16(vb[ch * 8 + 4], vb[ch * 8 + 5]);
                x.w = pack_bf16(vb[ch * 8 + 6], vb[ch * 8 + 7]);
                y.x = pack_bf16(vbg[ch * 8 + 0], vbg[ch * 8 + 1]);
                y.y = pack_bf16(vbg[ch * 8 + 2], vbg[ch * 8 + 3]);
                y.z = pack_bf16(vbg[ch * 8 + 4], vbg[ch * 8 + 5]);
                y.w = pack_bf16(vbg[ch * 8 + 6], vbg[ch * 8 + 7]);
                const uint32_t off = (uint32_t)(j * 128 + ((chunk ^ (j & 7)) << 4));
                st_shared_v4(sm + OFF_TB, off, x);
                st_shared_v4(sm + OFF_TBG, off, y);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- MMA 2 / 3: W^T = K^T (T diag(beta gamma))^T -> TM_P, U'^T = V^T (T diag(beta))^T -> TM_U ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16_ss(tbase + TM_P, smem_desc_sw128(s_tile + kk * 2048, 16384, 1024),
                            smem_desc_sw128(s_tbg + kk * 32, 16, 1024), id_w, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16_ss(tbase + TM_U, smem_desc_sw128(s_vtile + kk * 2048, v_lbo, 1024),
                            smem_desc_sw128(s_tb + kk * 32, 16, 1024), id_w, kk > 0);
            }
            mma_commit(&bar_mma);
        }
        ok = wait_all(&bar_mma, ph_mma, a, 3);
        ph_mma ^= 1;
        if (!ok) break;
        tc_fence_after();

        // ---- epilogue 2: -W^T (bf16, row = key index) and diag(gamma) Q ----
        {
            float v[64];
            tmem_ld32(tlane + TM_P, v);
            tmem_ld32(tlane + TM_P + 32, v + 32);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < C; ++j) v[j] = -v[j];
            write_row64_bf16(sm + OFF_WT, tid, v);
            if (!REPLAY) {
                const int i = tid >> 1, half = tid & 1;   // row i, key block `half`
                const uint8_t* qb = tile + half * 16384 + 8192;
                const float gi = s_gam[i];
#pragma unroll
                for (int col = 0; col < 64; ++col) v[col] = gi * bf16_at(qb, i, col);
                write_row64_bf16(sm + OFF_GQ + half * 8192, i, v);
            }
        }
        // ---- S epilogue: bf16 S_{c-1} for the operands, then S <- gamma_C S in TMEM ----
        {
            const float gC = s_gam[C - 1];
            uint8_t* sb = sm + OFF_SB;
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float v[32];
                tmem_ld32(tlane + TM_S + cb * 32, v);
                tmem_wait_ld();
                // columns [32 cb, 32 cb + 32) of key row tid -> dv block (cb / 2)
                uint8_t* blk = sb + (cb >> 1) * 16384;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const int chunk = (cb & 1) * 4 + ch;
                    uint4 x;
                    x.x = pack_bf16(v[ch * 8 + 0], v[ch * 8 + 1]);
                    x.y = pack_bf16(v[ch * 8 + 2], v[ch * 8 + 3]);
                    x.z = pack_bf16(v[ch * 8 + 4], v[ch * 8 + 5]);
                    x.w = pack_bf16(v[ch * 8 + 6], v[ch * 8 + 7]);
                    st_shared_v4(blk, (uint32_t)(tid * 128 + ((chunk ^ (tid & 7)) << 4)), x);
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= gC;
                tmem_st32(tlane + TM_S + cb * 32, v);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA U: U^T += S^T (-W^T);  prefill: O^T = S^T (gamma Q)^T ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                mma_bf16_ss(tbase + TM_U, smem_desc_sw128(s_sb + kk * 2048, 16384, 1024),
                            smem_desc_sw128(s_wt + kk * 2048, 16384, 1024), id_u, 1u);
            }
            if (!REPLAY) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    mma_bf16_ss(tbase + TM_O, smem_desc_sw128(s_sb + kk * 2048, 16384, 1024),
                                smem_desc_sw128(s_gq + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id_o1,
                                kk > 0);
                }
            }
            mma_commit(&bar_mma);
        }
        ok = wait_all(&bar_mma, ph_mma, a, 4);
        ph_mma ^= 1;
        if (!ok) break;
        tc_fence_after();

        // ---- epilogue U: diag(gamma_C / gamma) U (and U itself for the outputs) ----
        {
            float v[64];
            tmem_ld32(tlane + TM_U, v);
            tmem_ld32(tlane + TM_U + 32, v + 32);
            tmem_wait_ld();
            if (!REPLAY) write_row64_bf16(sm + OFF_UB, tid, v);
            const float g2C = s_g2[C - 1];
#pragma unroll
            for (int j = 0; j < C; ++j) v[j] *= exp2f(g2C - s_g2[j]);
            write_row64_bf16(sm + OFF_UT, tid, v);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA S: S += K^T U~ ;  prefill: O^T += U^T M^T ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16_ss(tbase + TM_S, smem_desc_sw128(s_tile + kk * 2048, 16384, 1024),
                            smem_desc_sw128(s_ut + kk * 32, 16, 1024), id_s, 1u);
            }
            if (!REPLAY) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    mma_bf16_ss(tbase + TM_O, smem_desc_sw128(s_ub + kk * 32, 16, 1024),
                                smem_desc_sw128(s_mb + kk * 32, 16, 1024), id_o2, 1u);
                }
            }
            mma_commit(&bar_mma);
        }
        ok = wait_all(&bar_mma, ph_mma, a, 5);
        ph_mma ^= 1;
        if (!ok) break;
        tc_fence_after();

        // ---- epilogue O: o[r0 + i, h, tid] for the chunk's real rows ----
        if (!REPLAY) {
            float v[64];
            tmem_ld32(tlane + TM_O, v);
            tmem_ld32(tlane + TM_O + 32, v + 32);
            tmem_wait_ld();
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o_out);
#pragma unroll
            for (int i = 0; i < C; ++i)
                if (i < nc) o[((r0 + i) * H + h) * (long long)D + tid] = __float2bfloat16_rn(v[i]);
        }
        tc_fence_before();
        __syncthreads();
    }

    // ---- final state (thread t = key row t) ----
    if (ok && a.state_out) {
        tc_fence_after();
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            float v[32];
            tmem_ld32(tlane + TM_S + cb * 32, v);
            tmem_wait_ld();
            float4* dst = reinterpret_cast<float4*>(a.state_out + state_base + (size_t)tid * D + cb * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

// ---- tensor maps ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [rows][H][128] bf16, box = 64 columns x 1 head x 64 rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int H, long long rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    if (rows < 1) rows = 1;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool chunk_tc_supported(int dtype, int dk, int dv) { return dtype == 1 && dk == 128 && dv == 128; }

cudaError_t launch_chunk_tc(const CallArgs& a, cudaStream_t stream) {
    if (a.units == 0) return cudaSuccess;
    if (!chunk_tc_supported(a.dtype, a.dk, a.dv)) return cudaErrorInvalidValue;
    TcParams p;
    p.a = a;
    p.rows_total = a.rows_total;
    CUtensorMap mk, mv, mq;
    if (!a.k || !a.v) return cudaErrorInvalidValue;
    if (!make_map(&mk, a.k, a.num_heads, a.rows_total) || !make_map(&mv, a.v, a.num_heads, a.rows_total))
        return cudaErrorInvalidValue;
    const bool replay = a.kind == kReplay;
    if (!make_map(&mq, replay ? a.k : a.q, a.num_heads, a.rows_total)) return cudaErrorInvalidValue;
    const uint32_t smem = (replay ? SMEM_REPLAY : SMEM_PREFILL) + 1024;
    static bool attr_set[2] = {false, false};
    if (replay) {
        if (!attr_set[0]) {
            cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return e;
            attr_set[0] = true;
        }
        chunk_tc_kernel<true><<<(unsigned)a.units, NT, smem, stream>>>(p, mk, mv, mq);
    } else {
        if (!attr_set[1]) {
            cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return e;
            attr_set[1] = true;
        }
        chunk_tc_kernel<false><<<(unsigned)a.units, NT, smem, stream>>>(p, mk, mv, mq);
    }
    return cudaGetLastError();
}

}  // namespace gdn
