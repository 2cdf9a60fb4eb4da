// gdn_replay.cu -- the state-only tail replay on tcgen05 tensor cores (bf16
// k/v, d_k = d_v = 128, fp32 state in tensor memory).
//
// Tail-Replay ("Tail-Replay: Escaping the Curse of Linear Attention in
// Prefix Caching for Hybrid LLMs", section "Mecanismos Principais", item
// "Reconstrucao de Estado Independente") rebuilds each Gated DeltaNet
// layer's state by replaying only the last R tokens of the matched prefix
// from a zero state:
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T.
// The replay runs 64 tokens at a time in the chunkwise WY / UT form (see the
// chunk helpers): A_ij = beta_i (gamma_i / gamma_j) k_i.k_j, T = (I + A)^-1,
// W = T diag(beta gamma) K, U' = T diag(beta) V, U = U' - W S0,
// S_C = gamma_C S0 + K^T diag(gamma_C / gamma) U.
// With E = diag(gamma_C / gamma), this kernel forms E W and E U' directly
// (E scales the rows of the bf16 T operands), so U~ = E U = E U' - (E W) S0
// reaches the state update without another pass over U.  U~ stays in tensor
// memory: the U epilogue writes it back as bf16 over its own columns, and the
// state update reads it from there as the A operand.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn_chunk_common.h"

namespace gdn {
namespace {

using namespace sm100;
using namespace chunk;

// ---------------------------------------------------------------------------
// Tail replay with two chunks in flight inside the CTA.
//
// The state-independent front of chunk c + 1 (A = strict_tril(...K K^T) and
// the UT inverse) runs on warps 0-3 while warps 4-7 finish chunk c's state
// chain: the U epilogue (U~ to bf16 in TMEM), the state update on the tensor
// core, and the TMA of chunk c + 2 into the tile slot that update frees.  Warps 6-7 first write the
// lower-right quarter of A, the only part of A outside columns 0-31.  Then all
// eight warps form T diag(beta), W and U', and -sigma W of chunk c + 1 and start
// its state product, then K K^T of chunk c + 2.  98 KB of shared memory, 256
// TMEM columns and at most 128 registers per thread, so two CTAs share an SM.
constexpr uint32_t BAR_CHAIN = 2;   // named barrier of warps 4-7 (the state chain)
constexpr uint32_t BAR_A = 4;       // warps 6-7 -> warps 2-3: their part of A is written

__global__ void __launch_bounds__(NT, 2)
replay_pipe_kernel(const TcParams p, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v) {
    using L = Layout<true>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // bar_w: W and U' (two issuers); bar_u: the state product and the next chunk's
    // K K^T (two issuers); bar_s: the state update (one issuer)
    __shared__ uint64_t bar_tile[2], bar_w, bar_u, bar_s;
    __shared__ uint32_t tmem_slot;
    __shared__ Gates s_gates[2];    // chunk c uses s_gates[c & 1]

    const CallArgs& a = p.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wh = warp >> 2;   // TMEM lane quarter; which half of the warps
    const int row = wq * 32 + lane;            // this thread's TMEM lane
    const Unit u = a.unit_list[blockIdx.x];
    const int b = u.seq, h = u.head, H = a.num_heads;
    if (!window_agrees(a, b)) {
        if (tid == 0) atomicOr(&a.ws->status, kStatusMismatch);
        return;
    }
    const Window w = a.windows[b];
    const int nchunks = (w.len + C - 1) / C;
    // debug build: the unit and its window lie inside the plan's extents (uniform)
    if (!index_ok(a.ws, b >= 0 && b < a.batch && h >= 0 && h < H && w.row0 >= 0 && w.len >= 0 &&
                            w.row0 + w.len <= a.rows_total))
        return;

    if (tid == 0) {
        mbar_init(&bar_tile[0], 1);
        mbar_init(&bar_tile[1], 1);
        mbar_init(&bar_w, 2);
        mbar_init(&bar_u, 2);
        mbar_init(&bar_s, 1);
        mbar_fence_init();
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_slot;
    const uint32_t tlane = tbase + ((uint32_t)(wq * 32) << 16);
    auto tile_of = [&](int cc) { return sm + L::OFF_TILE + (cc & 1) * L::TILE; };
    if (tid == 0) {   // both slots are free: chunks 0 and 1
        for (int cc = 0; cc < 2 && cc < nchunks; ++cc)
            issue_tiles<true>(tile_of(cc), &bar_tile[cc & 1], &map_k, &map_v, &map_k, h,
                              (int)(w.row0 + (long long)cc * C), false);
    }

    float* AT = reinterpret_cast<float*>(sm + L::OFF_AT);
    float* Xs = reinterpret_cast<float*>(sm + L::OFF_X);
    const uint32_t s_bu = smem_u32(sm + L::OFF_BU);
    const uint32_t s_tb = smem_u32(sm + L::OFF_TB), s_tbg = smem_u32(sm + L::OFF_TBG);
    const size_t state_base = ((size_t)b * H + h) * D * D;
    {   // zero state: TMEM lane dv holds column dv of S / sigma (a row of S^T)
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.0f;
        tmem_st32(tlane + TM_S + (2 * wh) * 32, v);
        tmem_st32(tlane + TM_S + (2 * wh + 1) * 32, v);
        tmem_wait_st();
    }
    float sigma = 1.0f;

    const uint32_t id_kk = idesc_bf16(64, 64, false, false);   // K K^T; row r in lane 32 (r/16) + r%16
    const uint32_t id_w = idesc_bf16(128, 64, true, false);    // K^T (T..)^T, V^T (T..)^T
    const uint32_t id_u = idesc_tf32(128, 64, false, false);   // S^T (-sigma W^T), A in TMEM
    const uint32_t id_s = idesc_bf16(128, 128, false, true);   // U~^T K, A (U~^T) in TMEM
    uint32_t ph_w = 0, ph_u = 0, ph_s = 0;
    bool ok = true;

    auto load_gates = [&](int cc, float& al, float& be) {
        al = 1.0f;
        be = 0.0f;
        if (tid < C && cc * C + tid < w.len) {
            const long long r = w.row0 + (long long)cc * C + tid;
            if (index_ok(a.ws, r < a.rows_total)) {
                al = a.alpha[r * H + h];
                be = a.beta[r * H + h];
            }
        }
    };
    auto tiles_ready = [&](int cc) -> bool {
        uint8_t* tile = tile_of(cc);
        if (!wait_all(&bar_tile[cc & 1], (cc >> 1) & 1, a, 1)) return false;
        const int ncc = min(C, w.len - cc * C);
        if (ncc < C) {   // padded tokens are identity transitions: zero their rows
            const int nrows = C - ncc;
            for (int e = tid; e < 4 * nrows * 8; e += NT) {
                const int t = e / (nrows * 8), rr = ncc + (e / 8) % nrows, ch = e % 8;
                st_shared_v4(tile + t * 8192, (uint32_t)(rr * 128 + ch * 16), make_uint4(0, 0, 0, 0));
            }
            fence_proxy_async_smem();
        }
        __syncthreads();
        return true;
    };
    auto issue_kk = [&](int cc) {
        const uint64_t dk0 = smem_desc_sw128(smem_u32(tile_of(cc)), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t d = desc_advance(dk0, (kk >> 2) * L::K_BLK + (kk & 3) * 32);
            mma_bf16_ss(tbase + TM_P, d, d, id_kk, kk > 0);
        }
    };

    // Epilogue 1 of chunk cc over the 32 columns [cb, cb + 32):
    // A = strict_tril(beta_i (gamma_i / gamma_j) K K^T), fp32 into AT.  The M = 64
    // accumulator keeps rows 16 wq .. 16 wq + 15 in the quarter's first 16 lanes; this
    // thread takes rows i0 = 16 wq + lane / 4 and i0 + 8, columns cb + 8 k + 2 (lane % 4)
    // + {0, 1}, k = 0..3.  Every gate factor is read before the first store to AT (a
    // store through AT may alias them for the compiler, which would then serialise each
    // load behind the previous store), and while the TMEM load is in flight.
    auto epi1_half = [&](int cc, int cb) {
        const Gates& Gn = s_gates[cc & 1];
        const bool fast = Gn.g2[C - 1] >= kFastGateFloor;
        float v[16];
        tmem_ld16x256b_x4(tlane + TM_P + cb, v);
        const int i0 = 16 * wq + (lane >> 2), jb = cb + 2 * (lane & 3);
        const float* colf = fast ? Gn.binv : Gn.g2;   // column factor: 2^-G_j, or G_j
        float2 cf[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) cf[k] = *reinterpret_cast<const float2*>(colf + jb + 8 * k);
        float gi[2], bi[2], rowf[2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int i = i0 + 8 * hf;
            gi[hf] = Gn.g2[i];
            bi[hf] = Gn.beta[i];
            rowf[hf] = bi[hf] * Gn.gam[i];
        }
        tmem_wait_ld();
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int i = i0 + 8 * hf;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int j = jb + 8 * k;
                float x0 = v[4 * k + 2 * hf], x1 = v[4 * k + 2 * hf + 1];
                if (fast) {
                    x0 *= rowf[hf] * cf[k].x;
                    x1 *= rowf[hf] * cf[k].y;
                } else {
                    x0 *= bi[hf] * exp2f(gi[hf] - cf[k].x);
                    x1 *= bi[hf] * exp2f(gi[hf] - cf[k].y);
                }
                x0 = (j < i) ? x0 : 0.0f;
                x1 = (j + 1 < i) ? x1 : 0.0f;
                *reinterpret_cast<float2*>(AT + i * LDT + j) = make_float2(x0, x1);
            }
        }
    };

    // ---- prologue: gates of chunk 0 (built) and 1 (registers), K K^T of chunk 0 ----
    float al_nxt, be_nxt;
    load_gates(0, al_nxt, be_nxt);
    if (tid < C) build_gates(s_gates[0], al_nxt, be_nxt, tid, lane);
    load_gates(1, al_nxt, be_nxt);
    if (nchunks > 0) {
        ok = tiles_ready(0);
        if (ok && (warp == 2 || warp == 3)) {
            tc_fence_after();
            if (elect_one()) {
                if (warp == 3) issue_kk(0);
                mma_commit(&bar_u);
            }
            __syncwarp();
        }
        if (ok) {
            ok = wait_all(&bar_u, ph_u, a, 2);
            ph_u ^= 1;
        }
    }

    // Iteration c: phase X overlaps chunk c's chain (c >= 0) with chunk c + 1's front;
    // phase Y finishes chunk c + 1's state-independent part and starts its state product.
    for (int c = -1; c < nchunks && ok; ++c) {
        const int cn = c + 1;
        const bool has_next = cn < nchunks;
        bool xok = true;
        tc_fence_after();
        if (warp < 4) {
            if (has_next) {
                // ---- epilogue 1 of chunk cn, columns 0-31 (warps 6-7 take rows 32-63 x
                //      columns 32-63; rows 0-31 have no entries there) ----
                epi1_half(cn, 0);
                __syncwarp();
                // the diagonal solve of block wq reads rows 16 wq .. 16 wq + 15; for wq >= 2
                // their columns 32-63 come from warps 6-7 (the later stages of the inverse
                // start after a barrier of warps 0-3 that follows this one)
                if (wq >= 2) named_sync(BAR_A, 128);
                // ---- T = (I + A)^-1 in place ----
                invert_unit_lower_inplace(AT, Xs, tid, BAR_INV);
            }
        } else {
            if (has_next && warp >= 6) {
                epi1_half(cn, 32);
                named_arrive(BAR_A, 128);
            }
        }
        if (warp >= 4 && c >= 0) {
            // ---- epilogue U of chunk c: U~ = diag(gamma_C / gamma) U / sigma_new into the
            //      chunk's V boxes (the row decay is already in U, through the rows of the T
            //      operands); the decay is folded into the TMEM state when sigma gets small ----
            Gates& G = s_gates[c & 1];
            uint8_t* tile = tile_of(c);
            float snew = sigma * G.gam[C - 1];
            if (snew < kRenormBelow) {   // uniform
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) {
                    float sv[32];
                    tmem_ld32(tlane + TM_S + cb * 32, sv);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 32; ++q) sv[q] *= snew;
                    tmem_st32(tlane + TM_S + cb * 32, sv);
                }
                tmem_wait_st();
                snew = 1.0f;
            }
            const float inv = 1.0f / snew;
            // U~^T as bf16 back into TMEM, two chunk rows per 32-bit column, over the first 32
            // columns of TM_U (half hf lands on columns 16 hf .. 16 hf + 15, which this thread
            // has read already): the A operand of the state update, with no trip through
            // shared memory
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float v[32];   // value dv = row, chunk rows [32 hf, 32 hf + 32)
                tmem_ld32(tlane + TM_U + 32 * hf, v);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) pk[q] = pack_bf16(v[2 * q] * inv, v[2 * q + 1] * inv);
                tmem_st16(tlane + TM_U + 16 * hf, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            named_sync(BAR_CHAIN, 128);
            // ---- S^T / sigma += U~^T K of chunk c; once it is done the slot takes chunk c + 2 ----
            if (warp == 4) {
                tc_fence_after();
                if (elect_one()) {
                    const uint32_t s_tile = smem_u32(tile);
                    const uint64_t db = smem_desc_sw128(s_tile, L::K_BLK, 1024);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(tbase + TM_S, tbase + TM_U + kk * 8, desc_advance(db, kk * 2048), id_s, 1u);
                    mma_commit(&bar_s);
                    if (mbar_wait_bounded(&bar_s, ph_s, kWaitNs)) {
                        if (c + 2 < nchunks)
                            issue_tiles<true>(tile, &bar_tile[c & 1], &map_k, &map_v, &map_k, h,
                                              (int)(w.row0 + (long long)(c + 2) * C), false);
                    } else {
                        report_timeout(a, 6);
                        xok = false;
                    }
                }
                __syncwarp();
            }
        }
        if (c >= 0) {   // every thread keeps the same running scale
            const float snew = sigma * s_gates[c & 1].gam[C - 1];
            sigma = snew < kRenormBelow ? 1.0f : snew;
            ph_s ^= 1;
        }
        ok = __syncthreads_and(xok) != 0;   // the state update of chunk c is done
        if (!ok || !has_next) break;

        // ---- phase Y, chunk cn: E T diag(beta), E T diag(beta gamma) in bf16 ----
        Gates& Gn = s_gates[cn & 1];
        const uint32_t s_tile_n = smem_u32(tile_of(cn));
        write_scaled_t<NT, false>(AT, Gn.beta, Gn.gam, sm + L::OFF_TB, sm + L::OFF_TBG, tid, 0, Gn.e);
        fence_proxy_async_smem();
        __syncthreads();
        // ---- (E W)^T = K^T (E T diag(beta gamma))^T -> TM_P and (E U')^T = V^T (E T diag(beta))^T -> TM_U ----
        if (warp == 0) {
            tc_fence_after();
            if (elect_one()) {
                const uint64_t da = smem_desc_sw128(s_tile_n, L::K_BLK, 1024);
                const uint64_t db = smem_desc_sw128(s_tbg, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ss(tbase + TM_P, desc_advance(da, kk * 2048), desc_advance(db, kk * 32), id_w, kk > 0);
                mma_commit(&bar_w);
            }
            __syncwarp();
        } else if (warp == 1) {
            tc_fence_after();
            if (elect_one()) {
                const uint64_t da = smem_desc_sw128(s_tile_n + L::V0, L::V_LBO, 1024);
                const uint64_t db = smem_desc_sw128(s_tb, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ss(tbase + TM_U, desc_advance(da, kk * 2048), desc_advance(db, kk * 32), id_w, kk > 0);
                mma_commit(&bar_w);
            }
            __syncwarp();
        }
        ok = wait_all(&bar_w, ph_w, a, 3);
        ph_w ^= 1;
        if (!ok) break;
        tc_fence_after();
        // ---- epilogue 2: BU[j][dk] = -sigma (E W)[j][dk] (fp32, K-major) ----
        {
            float v[32];   // key dk = row, chunk rows [32 wh, 32 wh + 32)
            tmem_ld32(tlane + TM_P + 32 * wh, v);
            tmem_wait_ld();
            uint8_t* bu = sm + L::OFF_BU + wq * 8192;
            const float ns = -sigma;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
                *reinterpret_cast<float*>(bu + sw128_offset_f32(32 * wh + jj, lane)) = ns * v[jj];
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- state product of chunk cn (warp 2) at once; K K^T of chunk cn + 1 (warp 3) once
        //      its tiles are in, while warps 0-1 build chunk cn + 1's gate factors ----
        if (warp == 2) {
            tc_fence_after();
            if (elect_one()) {
                const uint64_t db = smem_desc_sw128(s_bu, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 16; ++kk)
                    mma_tf32_ts(tbase + TM_U, tbase + TM_S + kk * 8,
                                desc_advance(db, (kk >> 2) * 8192 + (kk & 3) * 32), id_u, 1u);
                mma_commit(&bar_u);
            }
            __syncwarp();
        }
        // A full next chunk: warp 3 alone waits for its tiles (the next block-wide barrier
        // orders them for every later reader).  A partial one: the block zero-pads it first.
        // A tile timeout still waits for the state product below before the block leaves.
        const bool has_nn = cn + 1 < nchunks;
        const bool nn_partial = has_nn && w.len - (cn + 1) * C < C;   // uniform
        bool tok = true;
        if (nn_partial) tok = tiles_ready(cn + 1);
        if (warp == 3) {
            // the thread that sees the tiles arrive is the one that issues the MMA reading them
            bool t = true;
            if (elect_one()) {
                if (has_nn && !nn_partial) {
                    t = mbar_wait_bounded(&bar_tile[(cn + 1) & 1], ((cn + 1) >> 1) & 1, kWaitNs);
                    if (!t) report_timeout(a, 1);
                }
                tc_fence_after();
                if (t && tok && has_nn) issue_kk(cn + 1);
                mma_commit(&bar_u);
            }
            tok = __all_sync(0xffffffffu, t) && tok;
        } else if (tid < C && has_nn) {
            build_gates(s_gates[(cn + 1) & 1], al_nxt, be_nxt, tid, lane);
        }
        if (has_nn) load_gates(cn + 2, al_nxt, be_nxt);
        {   // wait_all, with warp 3's tile flag in the same vote
            const bool okw = mbar_wait_bounded(&bar_u, ph_u, kWaitNs);
            ok = __syncthreads_and(okw && tok) != 0;
            if (!ok && tid == 0) report_timeout(a, 4);
        }
        ph_u ^= 1;
    }

    // ---- final state: S[dk][dv] = sigma * TMEM[lane dv][dk] ----
    tc_fence_after();
    if (ok && a.state_out) {
#pragma unroll
        for (int cb = 2 * wh; cb < 2 * wh + 2; ++cb) {
            float v[32];
            tmem_ld32(tlane + TM_S + cb * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) a.state_out[state_base + (size_t)(cb * 32 + i) * D + row] = sigma * v[i];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 256);
    }
}

}  // namespace

cudaError_t launch_replay_tc(const CallArgs& a, cudaStream_t stream) {
    if (a.units == 0) return cudaSuccess;
    if (!chunk_tc_supported(a.dtype, a.dk, a.dv)) return cudaErrorInvalidValue;
    TcParams p;
    p.a = a;
    // a call with no rows to read (every window empty) still runs, to write the states;
    // its tile maps are never read, so any aligned address stands in for a null buffer
    const void* kb = a.k ? a.k : static_cast<const void*>(a.ws);
    const void* vb = a.v ? a.v : static_cast<const void*>(a.ws);
    CUtensorMap mk, mv;
    if (!make_tile_map(&mk, kb, a.num_heads, a.rows_total, a.rs_qk) ||
        !make_tile_map(&mv, vb, a.num_heads, a.rows_total, a.rs_v))
        return cudaErrorInvalidValue;
    static std::atomic<uint64_t> smem_set{0};
    const uint32_t smem = Layout<true>::BYTES + 1024;
    const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(replay_pipe_kernel), (int)smem, smem_set);
    if (e != cudaSuccess) return e;
    replay_pipe_kernel<<<(unsigned)a.units, NT, smem, stream>>>(p, mk, mv);
    return cudaGetLastError();
}

}  // namespace gdn
