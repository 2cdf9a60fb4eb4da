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
// U' = T diag(beta) V, U = U' - T diag(beta gamma) K S0,
// S_C = gamma_C S0 + K^T diag(gamma_C / gamma) U.
//
// This kernel groups the state-dependent term as T diag(beta gamma) (K S0):
// with E = diag(gamma_C / gamma), the state S = sigma S~ and P = K S~0,
//   E U = E U' - sigma (E T diag(beta gamma)) P,
//   S~_C = S~0 + K^T (E U) / (sigma gamma_C).
// P needs only the chunk's keys and the state, so it is formed on the tensor
// core as soon as the previous chunk's state update is done, while the
// chunk's T is still being built; once T is ready, E U is two MMAs into one
// accumulator (the P term, then E U' from V).  The serial part of a chunk is
// therefore: E U MMAs -> U epilogue -> state update -> P, with the next
// chunk's K K^T and A behind P and the chunk's inverse beside it.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn_chunk_common.h"

namespace gdn {
namespace {

using namespace sm100;
using namespace chunk;

// ---- shared memory (byte offsets from a 1 KB aligned base) ----
// K of a chunk stays from its K K^T (one iteration before the chunk's own)
// until its state update (one iteration after): three slots.  V stays only
// until its U' MMA (one slot).  AT holds A, then T in place, with the
// inverse's scratch in its unused upper-right quarter.  The inverse writes the
// T operands as their blocks become final: TB the bf16 E T diag(beta) (the B
// operand of U'), TG the fp32 -sigma' E T diag(beta gamma) (the B operand of
// the P term); the blocks above the diagonal are zeroed once and never written.
struct ReplayLayout {
    static constexpr uint32_t BOX = 8192;                   // 64 rows x 64 bf16 (128-byte swizzle)
    static constexpr uint32_t K_SLOT = 2 * BOX;             // [dk 0-63 | dk 64-127]
    static constexpr uint32_t OFF_K = 0;                    // chunk c in slot c % 3
    static constexpr uint32_t OFF_V = OFF_K + 3 * K_SLOT;   // [dv 0-63 | dv 64-127]
    static constexpr uint32_t OFF_AT = OFF_V + 2 * BOX;     // fp32 64 x LDT
    static constexpr uint32_t OFF_TB = OFF_AT + C * LDT * 4;   // bf16 [j][j'], 128-byte swizzled rows
    static constexpr uint32_t OFF_TG = OFF_TB + 8192;          // fp32 [j][j'], two 8 KB blocks of 32 columns
    static constexpr uint32_t BYTES = OFF_TG + 16384;
};
static_assert(ReplayLayout::OFF_TB % 1024 == 0 && ReplayLayout::OFF_TG == ReplayLayout::OFF_TB + 8192,
              "operands on 1 KB, TG right after TB");
static_assert(2 * (ReplayLayout::BYTES + 1024 + 1024 + 5120) <= 228 * 1024,
              "two replay CTAs per SM (dynamic + alignment + reserved + static)");

// TMEM columns: the state S~^T (fp32, lane = value row), then two 64-column
// regions with fixed roles.  TM_X holds E U of chunk c - 1 (M = 128, lane =
// value row), then U~ = E U / sigma in bf16 over its first 32 columns, then
// after the state update a bf16 copy of S~^T (two keys per column, the A
// operand of P), then K K^T of chunk c + 1 (M = 64) until its A epilogue, then
// E U of chunk c.  TM_Y holds P^T of chunk c = S~^T K^T (fp32, lane = value
// row), the A operand of the P term.
constexpr uint32_t TM_X = 128;
constexpr uint32_t TM_Y = 192;

constexpr uint32_t BAR_CHAIN = 2;   // named barrier of warps 4-7 (the state chain)

// ---------------------------------------------------------------------------
// Tail replay.  Iteration c = 0 .. nchunks (the last one only ends the chain):
//   phase X  warps 0-3 (front): T = (I + A)^-1 of chunk c (its A was written in
//                       the last phase X), writing the chunk's T operands as each
//                       block of T is final, once E U of chunk c - 1 has read the
//                       previous ones;
//            warps 4-7 (chain): wait for E U of chunk c - 1 and load chunk c's
//                       values into the slot its U' freed; the U epilogue (U~ to
//                       bf16 in TM_X), the state update with chunk c - 1's keys,
//                       the keys of chunk c + 2 into the slot they free, a bf16
//                       copy of the new state in TM_X, P of chunk c into TM_Y, and
//                       once P has read the copy, K K^T of chunk c + 1 into TM_X;
//            then all warps: A of chunk c + 1 from TM_X into AT.
//   phase Y  warp 2: the P term of chunk c, then U', into TM_X (E U of chunk c);
//                       warps 0-1 build the gates of chunk c + 2.  No barrier
//                       follows: the next phase X waits on the mbarriers of what
//                       it reads.
// 105 KB of shared memory, 256 TMEM columns and at most 128 registers per
// thread, so two CTAs share an SM.
__global__ void __launch_bounds__(NT, 2)
replay_pipe_kernel(const TcParams p, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v) {
    using RL = ReplayLayout;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // bar_k: keys of chunk c (slot c % 3); bar_v: values; bar_kk: K K^T; bar_s: the
    // state update; bar_p: P; bar_u: E U (the P term and U').  One issuer each.
    __shared__ uint64_t bar_k[3], bar_v, bar_kk, bar_s, bar_p, bar_u;
    __shared__ uint32_t tmem_slot;
    __shared__ Gates s_gates[3];    // chunk c uses s_gates[c % 3]
    __shared__ int s_abort;         // a wait outside the block-wide barriers gave up

    const CallArgs& a = p.a;
    record_call(a);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wh = warp >> 2;   // TMEM lane quarter; which half of the warps
    const int row = wq * 32 + lane;            // this thread's TMEM lane
    const Unit u = a.unit_list[blockIdx.x];
    const int b = u.seq, h = u.head, H = a.num_heads;
    if (!window_agrees(a, b)) {
        if (tid == 0) report_status(a, kStatusMismatch);
        return;
    }
    const Window w = a.windows[b];
    const int nchunks = (w.len + C - 1) / C;
    // debug build: the unit and its window lie inside the plan's extents (uniform)
    if (!index_ok(a, b >= 0 && b < a.batch && h >= 0 && h < H && w.row0 >= 0 && w.len >= 0 &&
                            w.row0 + w.len <= a.rows_total))
        return;

    if (tid == 0) {
        s_abort = 0;
        for (int i = 0; i < 3; ++i) mbar_init(&bar_k[i], 1);
        mbar_init(&bar_v, 1);
        mbar_init(&bar_kk, 1);
        mbar_init(&bar_s, 1);
        mbar_init(&bar_p, 1);
        mbar_init(&bar_u, 1);
        mbar_fence_init();
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, 256);
        tmem_relinquish();
    }
    float* AT = reinterpret_cast<float*>(sm + RL::OFF_AT);
    // the T operands' blocks above the diagonal stay zero (made visible to the tensor
    // core by the proxy fence before the first MMA that reads them)
    for (int e = tid; e < (8192 + 16384) / 16; e += NT)
        st_shared_v4(sm + RL::OFF_TB, (uint32_t)(e * 16), make_uint4(0, 0, 0, 0));
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_slot;
    const uint32_t tlane = tbase + ((uint32_t)(wq * 32) << 16);
    auto kslot = [&](int cc) { return sm + RL::OFF_K + (cc % 3) * RL::K_SLOT; };
    auto kbar = [&](int cc) { return &bar_k[cc % 3]; };
    auto kpar = [](int cc) { return (uint32_t)((cc / 3) & 1); };
    auto issue_k = [&](int cc) {
        uint8_t* dst = kslot(cc);
        const int r0 = (int)(w.row0 + (long long)cc * C);
        mbar_arrive_expect_tx(kbar(cc), RL::K_SLOT);
        tma_load_3d(dst, &map_k, kbar(cc), 0, h, r0);
        tma_load_3d(dst + RL::BOX, &map_k, kbar(cc), 64, h, r0);
    };
    auto issue_v = [&](int cc) {
        const int r0 = (int)(w.row0 + (long long)cc * C);
        mbar_arrive_expect_tx(&bar_v, 2 * RL::BOX);
        tma_load_3d(sm + RL::OFF_V, &map_v, &bar_v, 0, h, r0);
        tma_load_3d(sm + RL::OFF_V + RL::BOX, &map_v, &bar_v, 64, h, r0);
    };
    if (tid == 0) {
        for (int cc = 0; cc < 3 && cc < nchunks; ++cc) issue_k(cc);
        if (nchunks > 0) issue_v(0);
    }

    const uint32_t s_tg = smem_u32(sm + RL::OFF_TG), s_tb = smem_u32(sm + RL::OFF_TB);
    const uint32_t s_v = smem_u32(sm + RL::OFF_V);
    const size_t state_base = ((size_t)b * H + h) * D * D;
    {   // zero state: TMEM lane dv holds column dv of S / sigma (a row of S^T)
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.0f;
        tmem_st32(tlane + TM_S + (2 * wh) * 32, v);
        tmem_st32(tlane + TM_S + (2 * wh + 1) * 32, v);
        tmem_wait_st();
    }
    float sigma = 1.0f;   // the scale of the state entering chunk c - 1 (1 up to chunk 0)

    const uint32_t id_kk = idesc_bf16(64, 64, false, false);   // K K^T; row r in lane 32 (r/16) + r%16
    const uint32_t id_w = idesc_bf16(128, 64, true, false);    // V^T (E T diag(beta))^T
    const uint32_t id_t = idesc_tf32(128, 64, false, false);   // P^T (-sigma E T diag(beta gamma))^T, A in TMEM
    const uint32_t id_p = idesc_bf16(128, 64, false, false);   // P^T = S~^T K^T, A (bf16 S~^T) in TMEM
    const uint32_t id_s = idesc_bf16(128, 128, false, true);   // U~^T K, A (U~^T) in TMEM
    bool ok = true;

    auto load_gates = [&](int cc, float& al, float& be) {
        al = 1.0f;
        be = 0.0f;
        if (tid < C && cc * C + tid < w.len) {
            const long long r = w.row0 + (long long)cc * C + tid;
            if (index_ok(a, r < a.rows_total)) {
                al = a.alpha[r * H + h];
                be = a.beta[r * H + h];
            }
        }
    };
    auto nrows_of = [&](int cc) { return min(C, w.len - cc * C); };

    // Epilogue 1 of chunk cc over the 32 columns [cb, cb + 32) of its K K^T (in TM_X):
    // A = strict_tril(beta_i (gamma_i / gamma_j) K K^T), fp32 into AT.  The M = 64
    // accumulator keeps rows 16 wq .. 16 wq + 15 in the quarter's first 16 lanes; this
    // thread takes rows i0 = 16 wq + lane / 4 and i0 + 8, columns cb + 8 k + 2 (lane % 4)
    // + {0, 1}, k = 0..3.  Every gate factor is read before the first store to AT (a
    // store through AT may alias them for the compiler, which would then serialise each
    // load behind the previous store), and while the TMEM load is in flight.
    auto epi1_half = [&](int cc, int cb) {
        const Gates& Gn = s_gates[cc % 3];
        const bool fast = Gn.g2[C - 1] >= kFastGateFloor;
        float v[16];
        tmem_ld16x256b_x4(tlane + TM_X + cb, v);
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
    // A of chunk cc from its K K^T: warps 0-3 take columns 0-31 of their quarter's rows,
    // warps 6-7 columns 32-63 of rows 32-63 (rows 0-31 have no entries there); false if
    // the wait for K K^T ran out
    auto a_epilogue = [&](int cc) -> bool {
        if (warp >= 4 && warp < 6) return true;
        const bool t = mbar_wait_bounded(&bar_kk, cc & 1, kWaitNs);
        if (!t) report_timeout(a, 2);
        tc_fence_after();
        epi1_half(cc, warp < 4 ? 0 : 32);
        return t;
    };
    // zero the rows past the window of a partial chunk's key (bx = 0) or value slot,
    // with nth threads (index ct), after the tile has arrived
    auto zero_tail_rows = [&](uint8_t* slot, int nrows, int ct, int nth) {
        const int nz = C - nrows;
        for (int e = ct; e < 2 * nz * 8; e += nth) {
            const int bx = e / (nz * 8), rr = nrows + (e / 8) % nz, ch = e % 8;
            st_shared_v4(slot + bx * RL::BOX, (uint32_t)(rr * 128 + ch * 16), make_uint4(0, 0, 0, 0));
        }
    };
    auto issue_kk = [&](int cc) {
        const uint64_t dk0 = smem_desc_sw128(smem_u32(kslot(cc)), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t d = desc_advance(dk0, (kk >> 2) * RL::BOX + (kk & 3) * 32);
            mma_bf16_ss(tbase + TM_X, d, d, id_kk, kk > 0);
        }
    };

    // ---- prologue: gates of chunks 0 and 1, A of chunk 0 ----
    float al_nxt, be_nxt;
    load_gates(0, al_nxt, be_nxt);
    if (tid < C) build_gates(s_gates[0], al_nxt, be_nxt, tid, lane);
    load_gates(1, al_nxt, be_nxt);
    if (tid < C) build_gates(s_gates[1], al_nxt, be_nxt, tid, lane);
    load_gates(2, al_nxt, be_nxt);
    if (nchunks > 0) {
        bool t = true;
        if (nrows_of(0) < C) {
            t = mbar_wait_bounded(kbar(0), 0, kWaitNs);
            if (t) zero_tail_rows(kslot(0), nrows_of(0), tid, NT);
            else report_timeout(a, 1);
            fence_proxy_async_smem();
        }
        ok = __syncthreads_and(t) != 0;
        if (ok && warp == 0) {
            if (elect_one()) {
                bool tw = true;
                if (nrows_of(0) == C) {
                    tw = mbar_wait_bounded(kbar(0), 0, kWaitNs);
                    if (!tw) report_timeout(a, 1);
                }
                tc_fence_after();
                if (tw) issue_kk(0);
                mma_commit(&bar_kk);
            }
            __syncwarp();
        }
        if (ok) ok = a_epilogue(0);
    }
    tc_fence_before();
    ok = __syncthreads_and(ok) != 0;
    tc_fence_after();

    for (int c = 0; c <= nchunks && ok; ++c) {
        const bool has_cur = c < nchunks, has_prev = c >= 1, has_nx = c + 1 < nchunks;
        // the scale of the state entering chunk c, after chunk c - 1's update (the same
        // fp32 arithmetic in every thread); below 2^-40 it is folded into the state
        float snew = 1.0f, sig_c = sigma;
        bool fold = false;
        if (has_prev) {
            snew = sigma * s_gates[(c - 1) % 3].gam[C - 1];
            fold = snew < kRenormBelow;
            sig_c = fold ? 1.0f : snew;
        }
        bool xok = true;
        // =============================== phase X ===============================
        if (warp < 4) {
            if (has_cur) {
                // ---- T = (I + A)^-1 of chunk c in place, writing its T operands once the P
                //      term and U' of chunk c - 1 have read the previous ones ----
                const TOperandEmit<true> em{&s_gates[c % 3], -sig_c, sm + RL::OFF_TB, has_prev ? &bar_u : nullptr,
                                            (uint32_t)((c - 1) & 1), &a, &s_abort};
                invert_unit_lower_inplace<GDN_INV_SCRATCH_IN_AT>(AT, AT + 32, tid, BAR_INV, em);
                fence_proxy_async_smem();   // the T operands, for phase Y's MMAs
            }
        } else {
            const int ct = tid - 128;
            if (has_prev) {
                // ---- E U of chunk c - 1 is done: its U' has read the value slot ----
                bool t = mbar_wait_bounded(&bar_u, (c - 1) & 1, kWaitNs);
                if (!t) report_timeout(a, 4);
                xok = xok && t;
                tc_fence_after();
                if (warp == 4 && xok && has_cur) {
                    if (elect_one()) issue_v(c);
                    __syncwarp();
                }
                // ---- epilogue U of chunk c - 1: U~ = E U / sigma_new, bf16 back into TMEM over
                //      the first 32 columns of TM_X (half hf lands on columns 16 hf .. 16 hf + 15,
                //      which this thread has read already); the decay is folded into the TMEM
                //      state when sigma gets small ----
                if (fold) {   // uniform
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) {
                        float sv[32];
                        tmem_ld32(tlane + TM_S + cb * 32, sv);
                        tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < 32; ++q) sv[q] *= snew;
                        tmem_st32(tlane + TM_S + cb * 32, sv);
                    }
                }
                const float inv = fold ? 1.0f : 1.0f / snew;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float v[32];   // value dv = row, chunk rows [32 hf, 32 hf + 32)
                    tmem_ld32(tlane + TM_X + 32 * hf, v);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) pk[q] = pack_bf16(v[2 * q] * inv, v[2 * q + 1] * inv);
                    tmem_st16(tlane + TM_X + 16 * hf, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                xok = named_sync_and(BAR_CHAIN, 128, xok);
                // ---- S~^T += U~^T K of chunk c - 1 ----
                if (warp == 4) {
                    tc_fence_after();
                    if (elect_one()) {
                        if (xok) {
                            const uint64_t db = smem_desc_sw128(smem_u32(kslot(c - 1)), RL::BOX, 1024);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_bf16_ts(tbase + TM_S, tbase + TM_X + kk * 8, desc_advance(db, kk * 2048), id_s, 1u);
                        }
                        mma_commit(&bar_s);
                    }
                    __syncwarp();
                }
                // ---- every chain thread waits for the update; the keys of chunk c + 2 go into
                //      the slot chunk c - 1 frees; then the bf16 copy of this thread's lane of
                //      S~^T into TM_X (U~ is read), two keys per column ----
                t = xok && mbar_wait_bounded(&bar_s, (c - 1) & 1, kWaitNs);
                if (xok && !t) report_timeout(a, 6);
                tc_fence_after();
                if (warp == 4 && t && c + 2 < nchunks) {
                    if (elect_one()) issue_k(c + 2);
                    __syncwarp();
                }
                if (t && has_cur) {
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) {
                        float sv[32];
                        tmem_ld32(tlane + TM_S + cb * 32, sv);
                        tmem_wait_ld();
                        uint32_t pk[16];
#pragma unroll
                        for (int q = 0; q < 16; ++q) pk[q] = pack_bf16(sv[2 * q], sv[2 * q + 1]);
                        tmem_st16(tlane + TM_X + cb * 16, pk);
                    }
                    tmem_wait_st();
                }
                tc_fence_before();
                xok = named_sync_and(BAR_CHAIN, 128, t) && xok;
                // ---- P^T of chunk c = S~^T K_c^T into TM_Y (the P term of chunk c - 1 has
                //      read it) ----
                if (warp == 4 && has_cur) {
                    tc_fence_after();
                    if (elect_one()) {
                        if (xok) {
                            const uint64_t dk = smem_desc_sw128(smem_u32(kslot(c)), 16, 1024);
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                mma_bf16_ts(tbase + TM_Y, tbase + TM_X + kk * 8,
                                            desc_advance(dk, (kk >> 2) * RL::BOX + (kk & 3) * 32), id_p, kk > 0);
                        }
                        mma_commit(&bar_p);
                    }
                    __syncwarp();
                }
            }
            if (has_nx) {
                // ---- K K^T of chunk c + 1 into TM_X once P of chunk c has read the state copy
                //      there; a partial tile first gets its rows past the window zeroed ----
                if (nrows_of(c + 1) < C) {   // uniform
                    const bool t = mbar_wait_bounded(kbar(c + 1), kpar(c + 1), kWaitNs);
                    if (t) zero_tail_rows(kslot(c + 1), nrows_of(c + 1), ct, 128);
                    else report_timeout(a, 1);
                    fence_proxy_async_smem();
                    xok = named_sync_and(BAR_CHAIN, 128, t && xok);
                }
                if (warp == 4) {
                    tc_fence_after();
                    if (elect_one()) {
                        bool tw = xok;
                        if (tw && nrows_of(c + 1) == C) {
                            tw = mbar_wait_bounded(kbar(c + 1), kpar(c + 1), kWaitNs);
                            if (!tw) report_timeout(a, 1);
                        }
                        if (tw && has_prev) {
                            tw = mbar_wait_bounded(&bar_p, (c - 1) & 1, kWaitNs);
                            if (!tw) report_timeout(a, 3);
                        }
                        tc_fence_after();
                        if (tw) issue_kk(c + 1);
                        mma_commit(&bar_kk);
                        if (!tw) s_abort = 1;
                    }
                    __syncwarp();
                }
            }
            if (has_cur && nrows_of(c) < C) {   // a partial chunk's values, before its U'
                const bool t = mbar_wait_bounded(&bar_v, c & 1, kWaitNs);
                if (t) zero_tail_rows(sm + RL::OFF_V, nrows_of(c), ct, 128);
                else report_timeout(a, 1);
                fence_proxy_async_smem();
                xok = xok && t;
            }
        }
        // ---- A of chunk c + 1 (the front is done with AT, and K K^T is issued) ----
        tc_fence_before();
        xok = __syncthreads_and(xok) != 0;
        if (has_nx && xok) xok = a_epilogue(c + 1);
        if (has_prev) sigma = sig_c;
        tc_fence_before();
        ok = __syncthreads_and(xok && s_abort == 0) != 0;
        if (!ok || !has_cur) break;
        tc_fence_after();

        // =============================== phase Y ===============================
        if (warp == 2) {
            // ---- (E U)^T of chunk c into TM_X: P^T (-sigma E T diag(beta gamma))^T, then
            //      + V^T (E T diag(beta))^T ----
            if (elect_one()) {
                bool t = true;
                if (nrows_of(c) == C) {
                    t = mbar_wait_bounded(&bar_v, c & 1, kWaitNs);
                    if (!t) report_timeout(a, 1);
                }
                if (t && has_prev && !has_nx) {   // with a next chunk its K K^T waited for P
                    t = mbar_wait_bounded(&bar_p, (c - 1) & 1, kWaitNs);
                    if (!t) report_timeout(a, 3);
                }
                tc_fence_after();
                if (t && has_prev) {   // the state is zero before chunk 0
                    const uint64_t d2 = smem_desc_sw128(s_tg, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_tf32_ts(tbase + TM_X, tbase + TM_Y + kk * 8,
                                    desc_advance(d2, (kk >> 2) * 8192 + (kk & 3) * 32), id_t, kk > 0);
                }
                if (t) {
                    const uint64_t dv = smem_desc_sw128(s_v, RL::BOX, 1024);
                    const uint64_t dt = smem_desc_sw128(s_tb, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ss(tbase + TM_X, desc_advance(dv, kk * 2048), desc_advance(dt, kk * 32), id_w,
                                    (has_prev || kk > 0) ? 1u : 0u);
                }
                mma_commit(&bar_u);
                if (!t) s_abort = 1;
            }
            __syncwarp();
        } else if (tid < C && c + 2 < nchunks) {
            build_gates(s_gates[(c + 2) % 3], al_nxt, be_nxt, tid, lane);
        }
        if (c + 2 < nchunks) load_gates(c + 3, al_nxt, be_nxt);
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
    const uint32_t smem = ReplayLayout::BYTES + 1024;
    const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(replay_pipe_kernel), (int)smem, smem_set);
    if (e != cudaSuccess) return e;
    replay_pipe_kernel<<<(unsigned)a.units, NT, smem, stream>>>(p, mk, mv);
    return cudaGetLastError();
}

}  // namespace gdn
