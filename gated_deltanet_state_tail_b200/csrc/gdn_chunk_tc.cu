// gdn_chunk_tc.cu -- chunked gated-delta-rule prefill on tcgen05 tensor cores
// (bf16 q/k/v, d_k = d_v = 128, fp32 state in tensor memory), the fused
// replay + suffix, and the dispatch of the chunked path (the state-only
// replay kernels are in gdn_replay.cu and gdn_replay_ws.cu).
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
// This kernel groups the state term through P = K (S0 / sigma):
//   U = U' - sigma (T diag(beta gamma)) P,   O = M U + diag(sigma gamma) (Q (S0 / sigma))
// Every chunk contraction is a tcgen05.mma with M = 128 (the value dimension,
// or the 64 chunk rows of K stacked on 64 rows of Q) and accumulators in TMEM.
// The state lives in TMEM transposed (lane = value row) as S / sigma with a
// running scalar sigma, so the decay costs no pass over the state (sigma is
// folded back only when it gets small).  After each state update a bf16 copy
// of S / sigma goes into TMEM, the A operand of P and of the outputs' state
// term; the P term reads P from TMEM as a tf32 operand.  T is built from
// 16 x 16 diagonal inverses on CUDA cores and warp-level tf32 tensor-core
// products for the blocks below the diagonal, and the inverse writes the T
// operands as its blocks become final.
//
// Work: one CTA of 8 warps per (sequence, head) unit, chunks in order, two in
// flight: warps 0-3 build A and M of chunk c + 1 and invert T while warps 4-7
// finish chunk c (its state update, outputs and the next tile prefetch) and
// form P of chunk c + 1.  Warps w and w + 4 share TMEM lane quarter w (the only
// lanes a warp may read).  prefill_pipe_kernel runs the prefill with outputs
// and the fused replay + suffix (the replay window's chunks first, without
// outputs): 169 KB of shared memory, 512 TMEM columns, one CTA per SM.
#include <atomic>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn_chunk_common.h"

namespace gdn {
namespace {

using namespace sm100;
using namespace chunk;

// ---------------------------------------------------------------------------
// Prefill (and fused replay + suffix) with two chunks in flight per CTA.
// Iteration c (chunk cn = c + 1 is the next one):
//   phase X  warps 0-3 (front): A and M of chunk cn from [K; Q] K^T (TM_P), then
//                       T = (I + A)^-1, writing the chunk's T operands T diag(beta)
//                       (bf16) and -sigma' T diag(beta gamma) (fp32) as each block of
//                       T is final;
//            warps 4-7 (chain): chunk c's U epilogue, its state update and
//                       O = U M^T, the TMA of chunk c + 2, chunk c's outputs
//                       O + diag(sigma gamma) (Q S~) (the state term scaled per row
//                       in fp32); then a bf16 copy of the new state in TMEM, and,
//                       once the front has read TM_P, P = K S~ of chunk cn into TM_P
//                       and the outputs' state term Q S~ of chunk cn into TM_OS, both
//                       from the bf16 state copy and the chunk's own K and Q tiles.
//   phase Y  warp 2: U of chunk cn = P^T (-sigma' T diag(beta gamma))^T (tf32) + U'
//                       into TM_U; warp 3: [K; Q] K^T of chunk cn + 1 into TM_P once
//                       the P term has read it; warps 0-1: the gates of chunk cn + 1.
// 169 KB of shared memory, 512 TMEM columns, one CTA per SM.
constexpr uint32_t BAR_CHAIN = 2;   // named barrier of warps 4-7
constexpr uint32_t BAR_KK = 5;      // warps 0-3 -> warp 4: [K; Q] K^T in TM_P is read, P may overwrite it
constexpr uint32_t TM_SB = 384;     // 64 columns (prefill): bf16 S~^T, two keys per column
constexpr uint32_t TM_OS = 448;     // 64 columns (prefill): the outputs' state term (Q S~)^T
struct PipeLayout {
    static constexpr uint32_t TILE = TileLayout::TILE;       // [K0 | Q0 | K1 | Q1 | V0 | V1]
    static constexpr uint32_t OFF_TILE = 0;
    static constexpr uint32_t OFF_AT = 2 * TILE;                // fp32 A, then T (scratch in its upper right)
    static constexpr uint32_t OFF_TB = OFF_AT + C * LDT * 4;    // bf16 T diag(beta)
    static constexpr uint32_t OFF_TG = OFF_TB + 8192;           // fp32 -sigma T diag(beta gamma), K-major
    static constexpr uint32_t OFF_UB = OFF_TG + 16384;          // the output stage: bf16 O, two [i][dv] tiles
    static constexpr uint32_t OFF_MB = OFF_UB + 16384;          // two bf16 M [i][j], chunk c in c % 2
    static constexpr uint32_t BYTES = OFF_MB + 16384;
};
static_assert(PipeLayout::OFF_TB % 1024 == 0 && PipeLayout::OFF_TG == PipeLayout::OFF_TB + 8192 &&
                  PipeLayout::OFF_MB % 1024 == 0 && PipeLayout::OFF_UB % 1024 == 0,
              "operands and the output stage (a TMA source) on 1 KB, TG right after TB");
static_assert(PipeLayout::BYTES + 1024 <= 227 * 1024, "fits one CTA per SM");
static_assert(TM_OS + 64 <= 512, "TMEM map");

__global__ void __launch_bounds__(NT, 1)
prefill_pipe_kernel(const TcParams p, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_k0, const __grid_constant__ CUtensorMap map_v0,
                    const __grid_constant__ CUtensorMap map_o) {
    using L = TileLayout;
    using PL = PipeLayout;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // bar_tile: the tiles of chunk c (slot c % 2); bar_kk: [K; Q] K^T; bar_s: the state
    // update and O += U M^T; bar_p: P and the outputs' state term; bar_x: the P term;
    // bar_u: U (the P term and U').  One issuer each.
    __shared__ uint64_t bar_tile[2], bar_kk, bar_s, bar_p, bar_x, bar_u;
    __shared__ uint32_t tmem_slot;
    __shared__ Gates s_gates[2];    // chunk c uses s_gates[c & 1]

    const CallArgs& a = p.a;
    record_call(a);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wh = warp >> 2;
    const int row = wq * 32 + lane;
    const Unit u = a.unit_list[blockIdx.x];
    const int b = u.seq, h = u.head, H = a.num_heads;
    if (!window_agrees(a, b)) {
        if (tid == 0) report_status(a, kStatusMismatch);
        return;
    }
    // Chunk stream of this unit: the fused call's replay window first (cache rows, no
    // outputs), then the sequence's rows with outputs.
    const Window w = a.windows[b];
    const bool fused = a.windows0 != nullptr;
    Window w0;
    w0.row0 = 0;
    w0.len = 0;
    if (fused) w0 = a.windows0[b];
    const int nA = (w0.len + C - 1) / C;
    const int nchunks = nA + (w.len + C - 1) / C;
    // debug build: the unit and its row ranges lie inside the plan's extents (uniform)
    if (!index_ok(a, b >= 0 && b < a.batch && h >= 0 && h < H && w.row0 >= 0 && w.len >= 0 &&
                            w.row0 + w.len <= a.rows_total && w0.row0 >= 0 && w0.len >= 0 &&
                            w0.row0 + w0.len <= (fused ? a.rows_total0 : 0)))
        return;
    struct ChunkSrc {
        long long r0;
        int nc;
        bool out;
    };
    auto chunk_src = [&](int cc) -> ChunkSrc {
        if (cc < nA) return ChunkSrc{w0.row0 + (long long)cc * C, min(C, w0.len - cc * C), false};
        const int k = cc - nA;
        return ChunkSrc{w.row0 + (long long)k * C, min(C, w.len - k * C), true};
    };
    auto tile_of = [&](int cc) { return sm + PL::OFF_TILE + (cc & 1) * PL::TILE; };
    auto issue_chunk = [&](int cc) {
        const ChunkSrc cs = chunk_src(cc);
        if (cs.out)
            issue_tiles(tile_of(cc), &bar_tile[cc & 1], &map_k, &map_v, &map_q, h, (int)cs.r0, true);
        else
            issue_tiles(tile_of(cc), &bar_tile[cc & 1], &map_k0, &map_v0, &map_q, h, (int)cs.r0, false);
    };
    // the state entering chunk 0 is zero unless the call passes one (a fused call starts
    // from zero): then chunk 0 has no P term and no state term in its outputs
    const bool s0_zero = fused || a.state_in == nullptr;
    auto has_state_terms = [&](int cc) { return cc > 0 || !s0_zero; };

    if (tid == 0) {
        mbar_init(&bar_tile[0], 1);
        mbar_init(&bar_tile[1], 1);
        mbar_init(&bar_kk, 1);
        mbar_init(&bar_s, 1);
        mbar_init(&bar_p, 1);
        mbar_init(&bar_x, 1);
        mbar_init(&bar_u, 1);
        mbar_fence_init();
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
        tma_prefetch_desc(&map_q);
        if (fused) {
            tma_prefetch_desc(&map_k0);
            tma_prefetch_desc(&map_v0);
        }
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    // the T operands' blocks above the diagonal stay zero
    for (int e = tid; e < (8192 + 16384) / 16; e += NT)
        st_shared_v4(sm + PL::OFF_TB, (uint32_t)(e * 16), make_uint4(0, 0, 0, 0));
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_slot;
    const uint32_t tlane = tbase + ((uint32_t)(wq * 32) << 16);
    if (tid == 0) {   // both slots are free: chunks 0 and 1
        for (int cc = 0; cc < 2 && cc < nchunks; ++cc) issue_chunk(cc);
    }

    float* AT = reinterpret_cast<float*>(sm + PL::OFF_AT);
    const uint32_t s_tb = smem_u32(sm + PL::OFF_TB), s_tg = smem_u32(sm + PL::OFF_TG);
    const size_t state_base = ((size_t)b * H + h) * D * D;
    {   // initial state: TMEM lane dv holds column dv of S (a row of S^T)
        float v[32];
#pragma unroll
        for (int cb = 2 * wh; cb < 2 * wh + 2; ++cb) {
            if (a.state_in && !fused) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = a.state_in[state_base + (size_t)(cb * 32 + i) * D + row];
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.0f;
            }
            tmem_st32(tlane + TM_S + cb * 32, v);
        }
        tmem_wait_st();
    }
    float sigma = 1.0f;

    const uint32_t id_kk = idesc_bf16(128, 64, false, false);   // [K;Q] K^T
    const uint32_t id_w = idesc_bf16(128, 64, true, false);     // V^T (T diag(beta))^T
    const uint32_t id_t = idesc_tf32(128, 64, false, false);    // P^T (-sigma T diag(beta gamma))^T, A in TMEM
    const uint32_t id_p = idesc_bf16(128, 64, false, false);    // S~^T K^T and S~^T (sigma gamma Q)^T, A in TMEM
    const uint32_t id_s = idesc_bf16(128, 128, false, true);    // U~^T K, A in TMEM
    const uint32_t id_o2 = idesc_bf16(128, 64, false, false);   // U^T M^T, A (U^T) in TMEM
    uint32_t ph_u = 0, ph_s = 0, ph_p = 0, ph_x = 0;
    bool ok = true;

    auto load_gates = [&](int cc, float& al, float& be) {
        al = 1.0f;
        be = 0.0f;
        if (tid < C && cc < nchunks) {
            const ChunkSrc cs = chunk_src(cc);
            if (tid < cs.nc) {
                const float* pa = cc < nA ? a.alpha0 : a.alpha;
                const float* pb = cc < nA ? a.beta0 : a.beta;
                const long long r = cs.r0 + tid;
                if (index_ok(a, r < (cc < nA ? a.rows_total0 : a.rows_total))) {
                    al = pa[r * H + h];
                    be = pb[r * H + h];
                }
            }
        }
    };
    auto tiles_ready = [&](int cc) -> bool {
        uint8_t* tile = tile_of(cc);
        if (!wait_all(&bar_tile[cc & 1], (cc >> 1) & 1, a, 1)) return false;
        const int ncc = chunk_src(cc).nc;
        if (ncc < C) {   // padded tokens are identity transitions: zero their rows
            const int nrows = C - ncc;
            for (int e = tid; e < 6 * nrows * 8; e += NT) {
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
    if (fused && nA == 0 && a.state_mid) {   // empty window: the state at L is zero
#pragma unroll
        for (int cb = 2 * wh; cb < 2 * wh + 2; ++cb)
#pragma unroll
            for (int i = 0; i < 32; ++i) a.state_mid[state_base + (size_t)(cb * 32 + i) * D + row] = 0.0f;
    }

    // ---- prologue: gates of chunk 0 (built) and 1 (registers), [K; Q] K^T of chunk 0 ----
    float al_nxt, be_nxt;
    load_gates(0, al_nxt, be_nxt);
    if (tid < C) build_gates(s_gates[0], al_nxt, be_nxt, tid, lane);
    load_gates(1, al_nxt, be_nxt);
    if (nchunks > 0) {
        ok = tiles_ready(0);
        if (ok && warp == 3) {
            tc_fence_after();
            if (elect_one()) {
                issue_kk(0);
                mma_commit(&bar_kk);
            }
            __syncwarp();
        }
    }

    for (int c = -1; c < nchunks && ok; ++c) {
        const int cn = c + 1;
        const bool has_next = cn < nchunks;
        // P and the outputs' state term of chunk cn are formed in this phase X
        const bool st_next = has_next && has_state_terms(cn);
        bool xok = true;
        tc_fence_after();
        if (warp < 4) {
            if (has_next) {
                // ---- epilogue 1 of chunk cn: warps 0-1 hold K rows (lane = row), warps 2-3 the
                //      Q rows; A = strict_tril(beta_i (gamma_i / gamma_j) K K^T) (fp32, in AT) and
                //      M = tril((gamma_i / gamma_j) Q K^T) (bf16, MB[cn % 2]) ----
                {
                    const bool t = mbar_wait_bounded(&bar_kk, cn & 1, kWaitNs);
                    if (!t) report_timeout(a, 2);
                    xok = xok && t;
                    tc_fence_after();
                }
                Gates& Gn = s_gates[cn & 1];
                const bool outn = chunk_src(cn).out;
                const bool krow = wq < 2;
                if (krow || outn) {
                    const bool fast = Gn.g2[C - 1] >= kFastGateFloor;
                    const int i = krow ? row : row - C;
                    const float gi = Gn.g2[i];
                    const float bi = krow ? Gn.beta[i] : 1.0f;
                    const float rowf = bi * Gn.gam[i];
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        float v[32];
                        tmem_ld32(tlane + TM_P + 32 * hf, v);
                        tmem_wait_ld();
                        if (fast) {
                            const float4* binv = reinterpret_cast<const float4*>(Gn.binv + 32 * hf);
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float4 bv = binv[q];
                                v[4 * q] *= rowf * bv.x;
                                v[4 * q + 1] *= rowf * bv.y;
                                v[4 * q + 2] *= rowf * bv.z;
                                v[4 * q + 3] *= rowf * bv.w;
                            }
                        } else {
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) v[jj] *= bi * exp2f(gi - Gn.g2[32 * hf + jj]);
                        }
                        if (krow) {
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) v[jj] = (32 * hf + jj < i) ? v[jj] : 0.0f;
#pragma unroll
                            for (int jj = 0; jj < 32; jj += 4)
                                *reinterpret_cast<float4*>(AT + i * LDT + 32 * hf + jj) =
                                    make_float4(v[jj], v[jj + 1], v[jj + 2], v[jj + 3]);
                        } else {
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) v[jj] = (32 * hf + jj <= i) ? v[jj] : 0.0f;
                            write_row32_bf16(sm + PL::OFF_MB + (cn & 1) * 8192, i, 4 * hf, v);
                        }
                    }
                }
                if (st_next) {   // [K; Q] K^T is read: P of chunk cn may take TM_P
                    tc_fence_before();
                    named_arrive(BAR_KK, 160);
                }
                named_sync(BAR_INV, 128);   // every row of A is in before the inverse reads it
                // ---- T = (I + A)^-1 in place, writing the T operands of chunk cn scaled with the
                //      state's scale entering it ----
                float sig = sigma;
                if (c >= 0) {
                    const float sn = sigma * s_gates[c & 1].gam[C - 1];
                    sig = sn < kRenormBelow ? 1.0f : sn;
                }
                const TOperandEmit<false> em{&Gn, -sig, sm + PL::OFF_TB, nullptr, 0u, &a, nullptr};
                invert_unit_lower_inplace<GDN_INV_SCRATCH_IN_AT, TOperandEmit<false>, true>(AT, AT + 32, tid, BAR_INV,
                                                                                            em);
                fence_proxy_async_smem();   // the T operands, for phase Y's MMAs
            }
        } else {
            const int ct = tid - 128;   // this thread among the chain's 128
            if (c >= 0) {
                // ---- chain of chunk c: U~ (and U^T for the outputs), the state update and
                //      O += U M^T, then chunk c's outputs ----
                Gates& G = s_gates[c & 1];
                const ChunkSrc src = chunk_src(c);
                const bool outc = src.out;
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
                // U^T (for the outputs) and U~^T = U^T diag(e) / sigma (for the state update) as
                // bf16 in TMEM, two chunk rows per 32-bit column: the A operands of both MMAs
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float v[32];
                    tmem_ld32(tlane + TM_U + 32 * hf, v);
                    tmem_wait_ld();
                    uint32_t pk[16];
                    if (outc) {
#pragma unroll
                        for (int q = 0; q < 16; ++q) pk[q] = pack_bf16(v[2 * q], v[2 * q + 1]);
                        tmem_st16(tlane + TM_UB + 16 * hf, pk);
                    }
                    const float4* ev = reinterpret_cast<const float4*>(G.e + 32 * hf);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 e4 = ev[q];
                        pk[2 * q] = pack_bf16(v[4 * q] * (e4.x * inv), v[4 * q + 1] * (e4.y * inv));
                        pk[2 * q + 1] = pack_bf16(v[4 * q + 2] * (e4.z * inv), v[4 * q + 3] * (e4.w * inv));
                    }
                    tmem_st16(tlane + TM_UT + 16 * hf, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                named_sync(BAR_CHAIN, 128);
                if (warp == 4) {
                    tc_fence_after();
                    if (elect_one()) {
                        const uint32_t s_tile = smem_u32(tile);
                        const uint32_t s_mb = smem_u32(sm + PL::OFF_MB + (c & 1) * 8192);
                        const uint64_t db = smem_desc_sw128(s_tile, L::K_BLK, 1024);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16_ts(tbase + TM_S, tbase + TM_UT + kk * 8, desc_advance(db, kk * 2048), id_s, 1u);
                        if (outc) {   // O = U M^T; the state term is added in the epilogue
                            const uint64_t dmb = smem_desc_sw128(s_mb, 16, 1024);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_bf16_ts(tbase + TM_O, tbase + TM_UB + kk * 8, desc_advance(dmb, kk * 32), id_o2,
                                            kk > 0 ? 1u : 0u);
                        }
                        mma_commit(&bar_s);
                        if (mbar_wait_bounded(&bar_s, ph_s, kWaitNs)) {
                            if (c + 2 < nchunks) issue_chunk(c + 2);
                        } else {
                            report_timeout(a, 6);
                            xok = false;
                        }
                    }
                    __syncwarp();
                }
                const float sig_c = sigma;   // the scale of the state entering chunk c
                sigma = snew;
                if (ct == 0 && outc) bulk_wait_group_read0();   // the last chunk's output store has read the stage
                named_sync(BAR_CHAIN, 128);   // the state update (and O) of chunk c are complete
                tc_fence_after();
                if (outc) {
                    // outputs: stage O as bf16 in the UB region, two 8 KB tiles of 64 rows i by
                    // 64 values dv (128-byte rows, 16-byte pieces XOR-swizzled by i % 8: the TMA
                    // layout), then one TMA store per tile for a full chunk, or 16-byte stores of
                    // the chunk's rows for a partial one.  O^T (lane = value dim dv, column =
                    // chunk row i) is read in the 16x256b shape, whose registers are the
                    // fragments of 8 x 8 blocks [dv][i]; stmatrix .trans writes each block as 8
                    // rows i of 8 values dv.
                    const uint32_t s_stage = smem_u32(sm + PL::OFF_UB);
                    // the state term's row factors sigma gamma_i for this thread's rows
                    // i = 8 k + 2 (lane % 4) + {0, 1}
                    const bool st_c = has_state_terms(c);   // uniform
                    float2 sg[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float2 g = *reinterpret_cast<const float2*>(s_gates[c & 1].gam + 8 * k + 2 * (lane & 3));
                        sg[k] = make_float2(sig_c * g.x, sig_c * g.y);
                    }
#pragma unroll
                    for (int lh = 0; lh < 2; ++lh) {   // lanes 16 lh .. 16 lh + 15 of the quarter
                        float v[32];   // register 4k + e: dv = 16 lh + lane/4 + 8 (e/2), i = 8k + 2 (lane%4) + e%2
                        const uint32_t tq = tlane + ((uint32_t)(16 * lh) << 16);
                        tmem_ld16x256b_x8(tq + TM_O, v);
                        tmem_wait_ld();
                        if (st_c) {   // O = U M^T + diag(sigma gamma) Q S~, in two halves of the rows
#pragma unroll
                            for (int half = 0; half < 2; ++half) {
                                float w[16];
                                tmem_ld16x256b_x4(tq + TM_OS + 32 * half, w);
                                tmem_wait_ld();
#pragma unroll
                                for (int kh = 0; kh < 4; ++kh) {
                                    const int k = 4 * half + kh;
                                    v[4 * k + 0] += sg[k].x * w[4 * kh + 0];
                                    v[4 * k + 1] += sg[k].y * w[4 * kh + 1];
                                    v[4 * k + 2] += sg[k].x * w[4 * kh + 2];
                                    v[4 * k + 3] += sg[k].y * w[4 * kh + 3];
                                }
                            }
                        }
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const int v0 = 32 * wq + 16 * lh + 8 * hf;   // the blocks' first dv
#pragma unroll
                            for (int kg = 0; kg < 2; ++kg) {   // blocks i = 8k.., k = 4 kg + m
                                uint32_t r[4];
#pragma unroll
                                for (int m = 0; m < 4; ++m) {
                                    const int k = 4 * kg + m;
                                    r[m] = pack_bf16(v[4 * k + 2 * hf], v[4 * k + 2 * hf + 1]);
                                }
                                const int i = 32 * kg + 8 * (lane >> 3) + (lane & 7);   // this lane's row
                                stmatrix_x4_trans(s_stage + (uint32_t)((v0 >> 6) * 8192 + i * 128 +
                                                                       ((((v0 & 63) >> 3) ^ (i & 7)) << 4)),
                                                  r);
                            }
                        }
                    }
                    const bool tma_out = src.nc == C && index_ok(a, src.r0 + C <= a.rows_total);   // uniform
                    if (tma_out) fence_proxy_async_smem();   // the stage, for the TMA store
                    named_sync(BAR_CHAIN, 128);
                    if (tma_out) {
                        if (ct == 0) {
                            tma_store_3d(&map_o, s_stage, 0, h, (int)src.r0);
                            tma_store_3d(&map_o, s_stage + 8192, 64, h, (int)src.r0);
                            bulk_commit_group();
                        }
                    } else {
                        const uint8_t* stage = sm + PL::OFF_UB;
                        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o_out);
#pragma unroll
                        for (int k = 0; k < (C * D / 8) / 128; ++k) {   // 16-byte pieces: 16 per row
                            const int idx = ct + k * 128, i = idx >> 4, ch = idx & 15;
                            if (i < src.nc && index_ok(a, src.r0 + i < a.rows_total))
                                *reinterpret_cast<uint4*>(o + ((src.r0 + i) * H + h) * (long long)D + ch * 8) =
                                    *reinterpret_cast<const uint4*>(stage + (ch >> 3) * 8192 + i * 128 +
                                                                    (((ch & 7) ^ (i & 7)) << 4));
                        }
                    }
                }
                if (fused && c == nA - 1 && a.state_mid) {   // the state at L (chunk c is the window's last)
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) {
                        float v[32];
                        tmem_ld32(tlane + TM_S + cb * 32, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            a.state_mid[state_base + (size_t)(cb * 32 + i) * D + row] = sigma * v[i];
                    }
                }
            }
            if (st_next) {
                // ---- chunk cn's state terms from a bf16 copy of S~^T (TM_SB): P^T = S~^T K^T into
                //      TM_P once the front has read it, and, with outputs, (Q S~)^T = S~^T Q^T into
                //      TM_OS (chunk c's outputs have read it); the row factors sigma' gamma_i are
                //      applied in chunk cn's output epilogue ----
                const bool outn = chunk_src(cn).out;
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) {
                    float sv[32];
                    tmem_ld32(tlane + TM_S + cb * 32, sv);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) pk[q] = pack_bf16(sv[2 * q], sv[2 * q + 1]);
                    tmem_st16(tlane + TM_SB + cb * 16, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                named_sync(BAR_CHAIN, 128);
                if (warp == 4) {
                    named_sync(BAR_KK, 160);
                    tc_fence_after();
                    if (elect_one()) {
                        const uint64_t dk = smem_desc_sw128(smem_u32(tile_of(cn)), 16, 1024);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_bf16_ts(tbase + TM_P, tbase + TM_SB + kk * 8,
                                        desc_advance(dk, (kk >> 2) * L::K_BLK + (kk & 3) * 32), id_p, kk > 0);
                        if (outn) {   // (Q S~)^T of chunk cn from its Q tile
                            const uint64_t dq = smem_desc_sw128(smem_u32(tile_of(cn) + L::Q0), 16, 1024);
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                mma_bf16_ts(tbase + TM_OS, tbase + TM_SB + kk * 8,
                                            desc_advance(dq, (kk >> 2) * L::K_BLK + (kk & 3) * 32), id_p, kk > 0);
                        }
                        mma_commit(&bar_p);
                    }
                    __syncwarp();
                }
            }
        }
        if (c >= 0) {   // every thread keeps the same running scale
            const float snew = sigma * s_gates[c & 1].gam[C - 1];
            if (warp < 4) sigma = snew < kRenormBelow ? 1.0f : snew;   // warps 4-7 updated it above
            ph_s ^= 1;
        }
        ok = __syncthreads_and(xok) != 0;
        if (!ok || !has_next) break;

        // ---- phase Y, chunk cn: U = U' + P^T (-sigma T diag(beta gamma))^T (warp 2); [K; Q] K^T
        //      of chunk cn + 1 once the P term has read TM_P (warp 3); the gates of chunk cn + 1
        //      (warps 0-1).  A partial next chunk is zero-padded by the block first. ----
        const bool has_nn = cn + 1 < nchunks;
        const bool nn_partial = has_nn && chunk_src(cn + 1).nc < C;   // uniform
        bool tok = true;
        if (nn_partial) tok = tiles_ready(cn + 1);
        uint8_t* tile_n = tile_of(cn);
        const uint32_t s_tile_n = smem_u32(tile_n);
        if (warp == 2) {
            tc_fence_after();
            bool t = tok;
            if (elect_one()) {
                if (t && st_next) {
                    t = mbar_wait_bounded(&bar_p, ph_p, kWaitNs);
                    if (!t) report_timeout(a, 3);
                }
                tc_fence_after();
                if (t && st_next) {
                    const uint64_t dg = smem_desc_sw128(s_tg, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_tf32_ts(tbase + TM_U, tbase + TM_P + kk * 8, desc_advance(dg, (kk >> 2) * 8192 + (kk & 3) * 32),
                                    id_t, kk > 0);
                }
                mma_commit(&bar_x);
                if (t) {
                    const uint64_t da = smem_desc_sw128(s_tile_n + L::V0, L::V_LBO, 1024);
                    const uint64_t db = smem_desc_sw128(s_tb, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ss(tbase + TM_U, desc_advance(da, kk * 2048), desc_advance(db, kk * 32), id_w,
                                    (st_next || kk > 0) ? 1u : 0u);
                }
                mma_commit(&bar_u);
            }
            tok = __all_sync(0xffffffffu, t) && tok;
        } else if (warp == 3) {
            bool t = tok;
            if (elect_one()) {
                if (t && has_nn && !nn_partial) {
                    t = mbar_wait_bounded(&bar_tile[(cn + 1) & 1], ((cn + 1) >> 1) & 1, kWaitNs);
                    if (!t) report_timeout(a, 1);
                }
                if (t && has_nn) {   // the P term is done reading TM_P
                    t = mbar_wait_bounded(&bar_x, ph_x, kWaitNs);
                    if (!t) report_timeout(a, 5);
                }
                tc_fence_after();
                if (t && has_nn) issue_kk(cn + 1);
                if (has_nn) mma_commit(&bar_kk);
            }
            tok = __all_sync(0xffffffffu, t) && tok;
        } else if (warp < 2 && tid < C && has_nn) {
            build_gates(s_gates[(cn + 1) & 1], al_nxt, be_nxt, tid, lane);
        }
        if (has_nn) load_gates(cn + 2, al_nxt, be_nxt);
        {   // U of chunk cn is complete (its MMAs are done with the T operands and the tile)
            const bool okw = mbar_wait_bounded(&bar_u, ph_u, kWaitNs);
            ok = __syncthreads_and(okw && tok) != 0;
            if (!ok && tid == 0) report_timeout(a, 4);
        }
        ph_u ^= 1;
        ph_x ^= 1;
        if (st_next) ph_p ^= 1;
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
    if (tid == 128) bulk_wait_group0();   // the outputs' TMA stores are done before the CTA leaves
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    // resolved once (thread-safe static initialisation); null if the driver lacks it
    static const EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return static_cast<EncodeTiledFn>(nullptr);
    }();
    return fn;
}

}  // namespace

// [rows][H][128] bf16 with rows row_stride elements apart, box = 64 columns x 1 head
// x 64 rows, 128-byte swizzle.
bool make_tile_map(CUtensorMap* m, const void* base, int H, long long rows, long long row_stride) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    if (rows < 1) rows = 1;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)row_stride * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool chunk_tc_supported(int dtype, int dk, int dv) { return dtype == 1 && dk == 128 && dv == 128; }

cudaError_t launch_chunk_tc(const CallArgs& a, cudaStream_t stream) {
    if (a.units == 0) return cudaSuccess;
    if (!chunk_tc_supported(a.dtype, a.dk, a.dv)) return cudaErrorInvalidValue;
    // the state-only replay kernels unless outputs are asked for (a prefill, a fused replay
    // + suffix, or a replay that also emits the window's outputs): the two-CTA-per-SM
    // kernel, the fastest or as fast at every launch size measured (one to 296 units); the
    // warp-specialised kernel (one CTA per SM) and the cluster-pair kernel (two SMs per
    // unit) only when the descriptor pins them
    if (a.kind == kReplay && a.o_out == nullptr) {
        switch (a.replay_variant) {
            case kReplayWarpSpec: return launch_replay_ws(a, stream);
            case kReplayPair: return launch_replay_pair(a, stream);
            default: return launch_replay_tc(a, stream);
        }
    }
    TcParams p;
    p.a = a;
    // a call with no rows to read (every window empty) still runs, to write the states;
    // its tile maps are never read, so any aligned address stands in for a null buffer
    const void* kb = a.k ? a.k : static_cast<const void*>(a.ws);
    const void* vb = a.v ? a.v : static_cast<const void*>(a.ws);
    const void* qb = a.q ? a.q : static_cast<const void*>(a.ws);
    CUtensorMap mk, mv, mq;
    if (!make_tile_map(&mk, kb, a.num_heads, a.rows_total, a.rs_qk) ||
        !make_tile_map(&mv, vb, a.num_heads, a.rows_total, a.rs_v) ||
        !make_tile_map(&mq, qb, a.num_heads, a.rows_total, a.rs_qk))
        return cudaErrorInvalidValue;
    // fused replay + suffix: maps of the replayed cache rows (otherwise unused copies)
    CUtensorMap mk0 = mk, mv0 = mv;
    if (a.windows0) {
        const void* kb0 = a.k0 ? a.k0 : static_cast<const void*>(a.ws);
        const void* vb0 = a.v0 ? a.v0 : static_cast<const void*>(a.ws);
        if (!make_tile_map(&mk0, kb0, a.num_heads, a.rows_total0, a.rs_qk) ||
            !make_tile_map(&mv0, vb0, a.num_heads, a.rows_total0, a.rs_v))
            return cudaErrorInvalidValue;
    }
    static std::atomic<uint64_t> smem_set{0};
    const uint32_t smem = PipeLayout::BYTES + 1024;
    const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(prefill_pipe_kernel), (int)smem, smem_set);
    if (e != cudaSuccess) return e;
    // the outputs' map ([rows, H, 128] bf16, packed), stored into by whole full chunks
    CUtensorMap mo = mk;
    if (a.o_out && !make_tile_map(&mo, a.o_out, a.num_heads, a.rows_total, (long long)a.num_heads * D))
        return cudaErrorInvalidValue;
    prefill_pipe_kernel<<<(unsigned)a.units, NT, smem, stream>>>(p, mk, mv, mq, mk0, mv0, mo);
    return cudaGetLastError();
}

}  // namespace gdn
