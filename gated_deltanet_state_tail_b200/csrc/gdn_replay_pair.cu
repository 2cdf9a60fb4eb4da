// gdn_replay_pair.cu -- the state-only tail replay with every (sequence, head)
// unit on a cluster of two CTAs on two SMs (bf16 k/v, d_k = d_v = 128, fp32
// state in tensor memory).  Plans run it only when the descriptor pins it
// (GDN_KERNEL_CHUNKED_TC_PAIR).  Measured on B200 against the two-CTA-per-SM
// kernel (gdn_replay.cu) on launches of 16 to 74 units: 2-6 us slower on
// windows of up to 20 chunks (a cluster launch and its hand-offs cost about
// 2 us more, and its chain takes about 5 K cycles per chunk, near the other
// kernel's 5.4 K at one CTA per SM), within 1-7 % on 52-chunk windows.  It
// gives the same bits as the two-CTA kernel: the same operations in the
// same order.
//
// Tail-Replay ("Tail-Replay: Escaping the Curse of Linear Attention in
// Prefix Caching for Hybrid LLMs", section "Mecanismos Principais", item
// "Reconstrucao de Estado Independente") rebuilds each Gated DeltaNet
// layer's state by replaying only the last R tokens of the matched prefix
// from a zero state:
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T.
// The chunk algebra is that of the two-CTA-per-SM replay kernel
// (gdn_replay.cu): with E = diag(gamma_C / gamma), S = sigma S~ and P = K S~0,
//   E U = E U' - sigma (E T diag(beta gamma)) P,   S~_C = S~0 + K^T (E U) / (sigma gamma_C).
// What differs is where the work runs.  The state-independent part of a chunk
// (K K^T, A, T = (I + A)^-1 and the two T operands) runs on the front CTA; the
// state chain (the U epilogue, the state update, the bf16 state copy, P and
// E U) on the chain CTA.  The front hands each chunk's T operands (24 KB) to
// the chain with one bulk copy into the chain CTA's shared memory (distributed
// shared memory, one destination, no multicast) and runs up to two chunks
// ahead.  On one SM the inverse's warp-level MMAs wait behind the chain's
// tensor-core work; on an SM of its own the front keeps ahead of the chain,
// whose chunk is then its own latency chain, split over eight warps (the TMEM
// epilogues on four warps, as in the two-CTA kernel, made a chunk 20 % slower).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn_chunk_common.h"

namespace gdn {
namespace {

using namespace sm100;
using namespace chunk;

// ---- shared memory (byte offsets from a 1 KB aligned base; the same in both CTAs) ----
struct PairLayout {
    static constexpr uint32_t BOX = 8192;                    // 64 rows x 64 bf16 (128-byte swizzle)
    static constexpr uint32_t K_SLOT = 2 * BOX;              // [d 0-63 | d 64-127]
    static constexpr uint32_t OFF_K = 0;                     // both: keys of chunk c in slot c % 3
    static constexpr uint32_t OFF_V = OFF_K + 3 * K_SLOT;    // chain: values of chunk c in slot c % 2
    static constexpr uint32_t OPS = 24576;                   // TB (bf16, 8 KB), then TG (fp32, 16 KB)
    static constexpr uint32_t OFF_OPS = OFF_V + 2 * K_SLOT;  // T operands of chunk c in slot c % 2
                                                             // (front: staging; chain: received)
    static constexpr uint32_t OFF_AT = OFF_OPS + 2 * OPS;    // front: A, then T in place (fp32 64 x LDT)
    static constexpr uint32_t BYTES = OFF_AT + C * LDT * 4;
};
static_assert(PairLayout::OFF_OPS % 1024 == 0 && PairLayout::OPS % 1024 == 0, "operand slots on 1 KB");
static_assert(PairLayout::BYTES + 1024 + 1024 + 8192 <= 228 * 1024, "one pair CTA per SM");

// TMEM columns.  Front: K K^T of the chunk (M = 64), 64 columns.  Chain (256):
// the state S~^T (lane = value row), TM_X (E U of chunk c - 1, then U~ in bf16,
// then the bf16 copy of S~^T, then E U of chunk c) and TM_Y (P^T of chunk c).
constexpr uint32_t TM_S = 0;
constexpr uint32_t TM_X = 128;
constexpr uint32_t TM_Y = 192;

// ---------------------------------------------------------------------------
// One cluster of two CTAs per unit (grid = 2 x units): rank 0 the front, rank 1
// the chain.  Hand-offs between the two: bar_ops[s] in the chain (the chain arms
// it with the bytes it expects; the front's copy of chunk c's T operands into
// slot s = c % 2 completes them) and bar_free[s] in the front (the chain arrives
// once chunk c's operands are read, if chunk c + 2 will reuse the slot).  Every
// wait gives up after 1 s.  On the way out the chain waits for every copy the
// front issued, so no copy lands in a CTA that has left.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NT, 1)
replay_pair_kernel(const TcParams p, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v) {
    using PL = PairLayout;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar_k[3], bar_v[2], bar_ops[2], bar_free[2], bar_kk, bar_s, bar_p, bar_u, bar_drain;
    __shared__ uint32_t tmem_slot;
    __shared__ Gates s_gates[3];    // chunk c uses s_gates[c % 3]
    __shared__ int s_abort;         // a wait of a single issuing thread gave up
    __shared__ uint32_t s_copies;   // front: T-operand copies issued
    __shared__ uint32_t s_ops_seen; // chain: chunks whose T operands have arrived

    const CallArgs& a = p.a;
    record_call(a);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wh = warp >> 2;   // TMEM lane quarter; which half of the columns
    const int row = wq * 32 + lane;            // this thread's TMEM lane
    const bool front = cluster_ctarank() == 0;
    const Unit u = a.unit_list[blockIdx.x >> 1];
    const int b = u.seq, h = u.head, H = a.num_heads;
    // both CTAs of a pair take the same unit, so they leave here together
    if (!window_agrees(a, b)) {
        if (front && tid == 0) report_status(a, kStatusMismatch);
        return;
    }
    const Window w = a.windows[b];
    const int nchunks = (w.len + C - 1) / C;
    if (!index_ok(a, b >= 0 && b < a.batch && h >= 0 && h < H && w.row0 >= 0 && w.len >= 0 &&
                         w.row0 + w.len <= a.rows_total))
        return;

    if (tid == 0) {
        s_abort = 0;
        s_copies = 0;
        s_ops_seen = 0;
        for (int i = 0; i < 3; ++i) mbar_init(&bar_k[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_v[i], 1);
            mbar_init(&bar_ops[i], 1);
            mbar_init(&bar_free[i], 1);
        }
        mbar_init(&bar_kk, 1);
        mbar_init(&bar_s, 1);
        mbar_init(&bar_p, 1);
        mbar_init(&bar_u, 1);
        mbar_init(&bar_drain, 1);
        mbar_fence_init();
        tma_prefetch_desc(&map_k);
        if (!front) tma_prefetch_desc(&map_v);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, front ? 64u : 256u);
        tmem_relinquish();
    }
    float* AT = reinterpret_cast<float*>(sm + PL::OFF_AT);
    // front: the T operands' blocks above the diagonal stay zero in both staging
    // slots (the copies carry the zeros to the chain)
    if (front)
        for (int e = tid; e < (int)(2 * PL::OPS / 16); e += NT)
            st_shared_v4(sm + PL::OFF_OPS, (uint32_t)(e * 16), make_uint4(0, 0, 0, 0));
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_slot;
    const uint32_t tlane = tbase + ((uint32_t)(wq * 32) << 16);

    auto kslot = [&](int cc) { return sm + PL::OFF_K + (cc % 3) * PL::K_SLOT; };
    auto kbar = [&](int cc) { return &bar_k[cc % 3]; };
    auto kpar = [](int cc) { return (uint32_t)((cc / 3) & 1); };
    auto vslot = [&](int cc) { return sm + PL::OFF_V + (cc & 1) * PL::K_SLOT; };
    auto nrows_of = [&](int cc) { return min(C, w.len - cc * C); };
    auto issue_k = [&](int cc) {
        uint8_t* dst = kslot(cc);
        const int r0 = (int)(w.row0 + (long long)cc * C);
        mbar_arrive_expect_tx(kbar(cc), PL::K_SLOT);
        tma_load_3d(dst, &map_k, kbar(cc), 0, h, r0);
        tma_load_3d(dst + PL::BOX, &map_k, kbar(cc), 64, h, r0);
    };
    auto issue_v = [&](int cc) {
        uint8_t* dst = vslot(cc);
        const int r0 = (int)(w.row0 + (long long)cc * C);
        mbar_arrive_expect_tx(&bar_v[cc & 1], PL::K_SLOT);
        tma_load_3d(dst, &map_v, &bar_v[cc & 1], 0, h, r0);
        tma_load_3d(dst + PL::BOX, &map_v, &bar_v[cc & 1], 64, h, r0);
    };
    // gates of token `idx` of chunk cc (1 and 0 past the window)
    auto load_gates = [&](int cc, int idx, float& al, float& be) {
        al = 1.0f;
        be = 0.0f;
        if (idx >= 0 && idx < C && cc * C + idx < w.len) {
            const long long r = w.row0 + (long long)cc * C + idx;
            if (index_ok(a, r < a.rows_total)) {
                al = a.alpha[r * H + h];
                be = a.beta[r * H + h];
            }
        }
    };
    // zero the rows past the window of a partial chunk's key or value slot, after the tile arrived
    auto zero_tail_rows = [&](uint8_t* slot, int nrows) {
        const int nz = C - nrows;
        for (int e = tid; e < 2 * nz * 8; e += NT) {
            const int bx = e / (nz * 8), rr = nrows + (e / 8) % nz, ch = e % 8;
            st_shared_v4(slot + bx * PL::BOX, (uint32_t)(rr * 128 + ch * 16), make_uint4(0, 0, 0, 0));
        }
    };

    // the gates of chunks 0 and 1 (tokens = threads 0-63), then the loads of chunk 2
    float al_nxt, be_nxt;
    load_gates(0, tid, al_nxt, be_nxt);
    if (tid < C) build_gates(s_gates[0], al_nxt, be_nxt, tid, lane);
    load_gates(1, tid, al_nxt, be_nxt);
    if (tid < C) build_gates(s_gates[1], al_nxt, be_nxt, tid, lane);
    __syncthreads();

    // peer addresses: the front copies into the chain's operand slots and completes the
    // chain's bar_ops; the chain arrives on the front's bar_free and reads its s_copies
    const uint32_t peer = front ? 1u : 0u;
    const uint32_t peer_ops = mapa_shared(smem_u32(sm + PL::OFF_OPS), peer);
    const uint32_t peer_bar_ops0 = mapa_shared(smem_u32(&bar_ops[0]), peer);
    const uint32_t peer_bar_ops1 = mapa_shared(smem_u32(&bar_ops[1]), peer);
    const uint32_t peer_free0 = mapa_shared(smem_u32(&bar_free[0]), peer);
    const uint32_t peer_free1 = mapa_shared(smem_u32(&bar_free[1]), peer);
    const uint32_t peer_copies = mapa_shared(smem_u32(&s_copies), peer);

    // tile loads in flight are tracked so that they can be drained on the way out
    int k_issued = 0, v_issued = 0;
    if (tid == 0) {
        for (int cc = 0; cc < 3 && cc < nchunks; ++cc) issue_k(cc);
        k_issued = min(3, nchunks);
        if (!front) {
            for (int cc = 0; cc < 2 && cc < nchunks; ++cc) {
                issue_v(cc);
                mbar_arrive_expect_tx(&bar_ops[cc], PL::OPS);   // armed before the front may copy
            }
            v_issued = min(2, nchunks);
        }
    }
    // both CTAs' barriers are initialised and the chain's first two operand phases armed
    cluster_sync();

    const uint32_t id_kk = idesc_bf16(64, 64, false, false);   // K K^T; row r in lane 32 (r/16) + r%16
    const uint32_t id_w = idesc_bf16(128, 64, true, false);    // V^T (E T diag(beta))^T
    const uint32_t id_t = idesc_tf32(128, 64, false, false);   // P^T (-sigma E T diag(beta gamma))^T, A in TMEM
    const uint32_t id_p = idesc_bf16(128, 64, false, false);   // P^T = S~^T K^T, A (bf16 S~^T) in TMEM
    const uint32_t id_s = idesc_bf16(128, 128, false, true);   // U~^T K, A (U~^T) in TMEM
    bool ok = true;
    float sigma = 1.0f;   // the scale of the state entering the current chunk

    if (front) {
        // =============================== front ===============================
        const int gi = tid - 192;   // warps 6-7 build the gates of chunk c + 2 (token gi)
        load_gates(2, gi, al_nxt, be_nxt);
        for (int c = 0; c < nchunks; ++c) {
            float sig_c = sigma;
            if (c >= 1) {   // the same fp32 arithmetic as the chain's
                const float snew = sigma * s_gates[(c - 1) % 3].gam[C - 1];
                sig_c = snew < kRenormBelow ? 1.0f : snew;
            }
            // ---- keys of chunk c (a partial tile first gets its rows past the window
            //      zeroed), then K K^T ----
            bool t = true;
            if (nrows_of(c) < C) {   // uniform
                t = mbar_wait_bounded(kbar(c), kpar(c), kWaitNs);
                if (t) zero_tail_rows(kslot(c), nrows_of(c));
                else report_timeout(a, 1);
                fence_proxy_async_smem();
            }
            ok = __syncthreads_and(t) != 0;
            if (!ok) break;
            if (warp == 0) {
                tc_fence_after();
                if (elect_one()) {
                    bool tw = true;
                    if (nrows_of(c) == C) {
                        tw = mbar_wait_bounded(kbar(c), kpar(c), kWaitNs);
                        if (!tw) report_timeout(a, 1);
                    }
                    tc_fence_after();
                    if (tw) {
                        const uint64_t dk0 = smem_desc_sw128(smem_u32(kslot(c)), 16, 1024);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t d = desc_advance(dk0, (kk >> 2) * PL::BOX + (kk & 3) * 32);
                            mma_bf16_ss(tbase, d, d, id_kk, kk > 0);
                        }
                    }
                    mma_commit(&bar_kk);
                    if (!tw) s_abort = 1;
                }
                __syncwarp();
            }
            // ---- A = strict_tril(beta_i (gamma_i / gamma_j) K K^T) into AT: warps 0-3 take
            //      columns 0-31 of their quarter's 16 rows, warps 6-7 columns 32-63 of rows
            //      32-63 (rows 0-31 have no entries there); the same arithmetic as the
            //      two-CTA kernel's ----
            if (warp < 4 || warp >= 6) {
                t = mbar_wait_bounded(&bar_kk, c & 1, kWaitNs);
                if (!t) report_timeout(a, 2);
                tc_fence_after();
                const int cb = warp < 4 ? 0 : 32;
                const Gates& Gn = s_gates[c % 3];
                const bool fast = Gn.g2[C - 1] >= kFastGateFloor;
                float v[16];
                tmem_ld16x256b_x4(tlane + cb, v);
                const int i0 = 16 * wq + (lane >> 2), jb = cb + 2 * (lane & 3);
                const float* colf = fast ? Gn.binv : Gn.g2;
                float2 cf[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) cf[k] = *reinterpret_cast<const float2*>(colf + jb + 8 * k);
                float gi2[2], bi[2], rowf[2];
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int i = i0 + 8 * hf;
                    gi2[hf] = Gn.g2[i];
                    bi[hf] = Gn.beta[i];
                    rowf[hf] = bi[hf] * Gn.gam[i];
                }
                tmem_wait_ld();
                if (t) {
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
                                x0 *= bi[hf] * exp2f(gi2[hf] - cf[k].x);
                                x1 *= bi[hf] * exp2f(gi2[hf] - cf[k].y);
                            }
                            x0 = (j < i) ? x0 : 0.0f;
                            x1 = (j + 1 < i) ? x1 : 0.0f;
                            *reinterpret_cast<float2*>(AT + i * LDT + j) = make_float2(x0, x1);
                        }
                    }
                }
            }
            tc_fence_before();
            ok = __syncthreads_and(t && s_abort == 0) != 0;
            if (!ok) break;
            tc_fence_after();
            // the key slot is read: chunk c + 3's keys go there
            if (tid == 0 && c + 3 < nchunks) {
                issue_k(c + 3);
                k_issued = c + 4;
            }
            if (warp < 4) {
                // ---- T = (I + A)^-1 of chunk c in place, its T operands into staging slot
                //      c % 2 once the chain has read chunk c - 2's from its own slot ----
                uint8_t* stg = sm + PL::OFF_OPS + (c & 1) * PL::OPS;
                bool tf = true;
                if (c >= 2) {
                    tf = mbar_wait_bounded_cluster(&bar_free[c & 1], (uint32_t)(((c - 2) >> 1) & 1), kWaitNs);
                    if (!tf) report_timeout(a, 9);
                }
                tf = named_sync_and(BAR_INV, 128, tf);
                if (tf) {
                    const TOperandEmit<true> em{&s_gates[c % 3], -sig_c, stg, nullptr, 0u, &a, &s_abort};
                    invert_unit_lower_inplace<GDN_INV_SCRATCH_IN_AT>(AT, AT + 32, tid, BAR_INV, em);
                    fence_proxy_async_smem();   // the operands, for the bulk copy
                    named_sync(BAR_INV, 128);
                    if (tid == 0) {
                        bulk_copy_to_peer(peer_ops + (uint32_t)(c & 1) * PL::OPS, smem_u32(stg), PL::OPS,
                                          (c & 1) ? peer_bar_ops1 : peer_bar_ops0);
                        s_copies = (uint32_t)(c + 1);
                    }
                } else if (tid == 0) {
                    s_abort = 1;
                }
            } else if (warp >= 6 && c + 2 < nchunks) {
                // ---- the gates of chunk c + 2, into the slot chunk c - 1 used ----
                build_gates(s_gates[(c + 2) % 3], al_nxt, be_nxt, gi, gi & 31);
            }
            if (c + 2 < nchunks) load_gates(c + 3, gi, al_nxt, be_nxt);
            if (c >= 1) sigma = sig_c;
        }
        // (the next iteration's first barrier orders the inverse's last reads of AT before
        // the next A epilogue's writes)
    } else {
        // =============================== chain ===============================
        const int gi = tid - 64;   // warps 2-3 build the gates of chunk c + 2 (token gi)
        load_gates(2, gi, al_nxt, be_nxt);
        {   // zero state: TMEM lane dv holds column dv of S / sigma (a row of S^T)
            float z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) z[i] = 0.0f;
            tmem_st32(tlane + TM_S + (2 * wh) * 32, z);
            tmem_st32(tlane + TM_S + (2 * wh + 1) * 32, z);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        const uint32_t s_ops = smem_u32(sm + PL::OFF_OPS);
        for (int c = 0; c <= nchunks; ++c) {
            const bool has_cur = c < nchunks, has_prev = c >= 1;
            // the scale of the state entering chunk c, after chunk c - 1's update (the same
            // fp32 arithmetic in every thread and in the front); below 2^-40 it is folded into
            // the state
            float snew = 1.0f, sig_c = sigma;
            bool fold = false;
            if (has_prev) {
                snew = sigma * s_gates[(c - 1) % 3].gam[C - 1];
                fold = snew < kRenormBelow;
                sig_c = fold ? 1.0f : snew;
            }
            bool t = true;
            if (has_prev) {
                // ---- E U of chunk c - 1 is done: its U' has read the value slot and its
                //      P term the operand slot, which chunk c + 1 may now take ----
                t = mbar_wait_bounded(&bar_u, (c - 1) & 1, kWaitNs);
                if (!t) report_timeout(a, 4);
                tc_fence_after();
                if (tid == 0 && t && c + 1 < nchunks) {
                    mbar_arrive_expect_tx(&bar_ops[(c + 1) & 1], PL::OPS);
                    mbar_arrive_peer((c + 1) & 1 ? peer_free1 : peer_free0);
                    issue_v(c + 1);
                    v_issued = c + 2;
                }
                // ---- U epilogue of chunk c - 1: U~ = E U / sigma_new in bf16; warp half wh
                //      takes chunk rows [32 wh, 32 wh + 32) and writes them to columns
                //      32 wh .. 32 wh + 15 of TM_X (its own, already read); the decay is
                //      folded into the TMEM state when sigma gets small ----
                if (fold) {   // uniform
#pragma unroll
                    for (int cb = 2 * wh; cb < 2 * wh + 2; ++cb) {
                        float sv[32];
                        tmem_ld32(tlane + TM_S + cb * 32, sv);
                        tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < 32; ++q) sv[q] *= snew;
                        tmem_st32(tlane + TM_S + cb * 32, sv);
                    }
                }
                const float inv = fold ? 1.0f : 1.0f / snew;
                {
                    float v[32];
                    tmem_ld32(tlane + TM_X + 32 * wh, v);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) pk[q] = pack_bf16(v[2 * q] * inv, v[2 * q + 1] * inv);
                    tmem_st16(tlane + TM_X + 32 * wh, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                ok = __syncthreads_and(t && s_abort == 0) != 0;
                if (!ok) break;
                // ---- S~^T += U~^T K of chunk c - 1 (U~'s k-steps 0-1 at columns 0-15,
                //      2-3 at 32-47) ----
                if (warp == 0) {
                    tc_fence_after();
                    if (elect_one()) {
                        bool tw = mbar_wait_bounded(kbar(c - 1), kpar(c - 1), kWaitNs);
                        if (!tw) report_timeout(a, 1);
                        tc_fence_after();
                        if (tw) {
                            const uint64_t db = smem_desc_sw128(smem_u32(kslot(c - 1)), PL::BOX, 1024);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_bf16_ts(tbase + TM_S, tbase + TM_X + (kk >> 1) * 32 + (kk & 1) * 8,
                                            desc_advance(db, kk * 2048), id_s, 1u);
                        }
                        mma_commit(&bar_s);
                        if (!tw) s_abort = 1;
                    }
                    __syncwarp();
                }
                // ---- every thread waits for the update; the keys of chunk c + 2 go into
                //      the slot chunk c - 1 frees; then the bf16 copy of this thread's lane of
                //      S~^T into TM_X, warp half wh taking key blocks 2 wh and 2 wh + 1 ----
                t = mbar_wait_bounded(&bar_s, (c - 1) & 1, kWaitNs);
                if (!t) report_timeout(a, 6);
                tc_fence_after();
                if (tid == 0 && t && c + 2 < nchunks) {
                    issue_k(c + 2);
                    k_issued = c + 3;
                }
                if (t && has_cur) {
#pragma unroll
                    for (int cb = 2 * wh; cb < 2 * wh + 2; ++cb) {
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
                ok = __syncthreads_and(t && s_abort == 0) != 0;
                if (!ok) break;
                tc_fence_after();
                sigma = sig_c;
            }
            if (!has_cur) break;
            // ---- a partial chunk's keys, then its values, get their rows past the window
            //      zeroed before any MMA reads them ----
            if (nrows_of(c) < C) {   // uniform
                t = mbar_wait_bounded(kbar(c), kpar(c), kWaitNs);
                if (t) t = mbar_wait_bounded(&bar_v[c & 1], (uint32_t)((c >> 1) & 1), kWaitNs);
                if (t) {
                    zero_tail_rows(kslot(c), nrows_of(c));
                    zero_tail_rows(vslot(c), nrows_of(c));
                } else {
                    report_timeout(a, 1);
                }
                fence_proxy_async_smem();
                ok = __syncthreads_and(t) != 0;
                if (!ok) break;
            }
            if (warp == 0) {
                tc_fence_after();
                if (elect_one()) {
                    bool tw = true;
                    if (has_prev) {
                        // ---- P^T of chunk c = S~^T K_c^T into TM_Y ----
                        if (nrows_of(c) == C) {
                            tw = mbar_wait_bounded(kbar(c), kpar(c), kWaitNs);
                            if (!tw) report_timeout(a, 1);
                        }
                        tc_fence_after();
                        if (tw) {
                            const uint64_t dk = smem_desc_sw128(smem_u32(kslot(c)), 16, 1024);
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                mma_bf16_ts(tbase + TM_Y, tbase + TM_X + kk * 8,
                                            desc_advance(dk, (kk >> 2) * PL::BOX + (kk & 3) * 32), id_p, kk > 0);
                        }
                        mma_commit(&bar_p);
                    }
                    // ---- (E U)^T of chunk c into TM_X once the values, the T operands and
                    //      P (which read the state copy there) are in: P^T
                    //      (-sigma E T diag(beta gamma))^T, then + V^T (E T diag(beta))^T ----
                    if (tw && nrows_of(c) == C) {
                        tw = mbar_wait_bounded(&bar_v[c & 1], (uint32_t)((c >> 1) & 1), kWaitNs);
                        if (!tw) report_timeout(a, 1);
                    }
                    if (tw) {
                        tw = mbar_wait_bounded(&bar_ops[c & 1], (uint32_t)((c >> 1) & 1), kWaitNs);
                        if (tw) s_ops_seen = (uint32_t)(c + 1);
                        else report_timeout(a, 7);
                    }
                    if (tw && has_prev) {
                        tw = mbar_wait_bounded(&bar_p, (c - 1) & 1, kWaitNs);
                        if (!tw) report_timeout(a, 3);
                    }
                    tc_fence_after();
                    const uint32_t s_tb = s_ops + (uint32_t)(c & 1) * PL::OPS, s_tg = s_tb + 8192;
                    if (tw && has_prev) {   // the state is zero before chunk 0
                        const uint64_t d2 = smem_desc_sw128(s_tg, 16, 1024);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_tf32_ts(tbase + TM_X, tbase + TM_Y + kk * 8,
                                        desc_advance(d2, (kk >> 2) * 8192 + (kk & 3) * 32), id_t, kk > 0);
                    }
                    if (tw) {
                        const uint64_t dv = smem_desc_sw128(smem_u32(vslot(c)), PL::BOX, 1024);
                        const uint64_t dt = smem_desc_sw128(s_tb, 16, 1024);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16_ss(tbase + TM_X, desc_advance(dv, kk * 2048), desc_advance(dt, kk * 32), id_w,
                                        (has_prev || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&bar_u);
                    if (!tw) s_abort = 1;
                }
                __syncwarp();
            } else if (warp >= 2 && warp < 4 && c + 2 < nchunks) {
                // ---- the gates of chunk c + 2, into the slot chunk c - 1 used ----
                build_gates(s_gates[(c + 2) % 3], al_nxt, be_nxt, gi, gi & 31);
            }
            if (c + 2 < nchunks) load_gates(c + 3, gi, al_nxt, be_nxt);
        }
        // ---- final state: S[dk][dv] = sigma * TMEM[lane dv][dk] ----
        tc_fence_after();
        if (ok && a.state_out) {
            const size_t state_base = ((size_t)b * H + h) * D * D;
#pragma unroll
            for (int cb = 2 * wh; cb < 2 * wh + 2; ++cb) {
                float v[32];
                tmem_ld32(tlane + TM_S + cb * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) a.state_out[state_base + (size_t)(cb * 32 + i) * D + row] = sigma * v[i];
            }
        }
    }

    // ---- the way out: drain this CTA's MMAs and tile loads, then, once the front has
    //      issued its last copy, let the chain take every copy aimed at it ----
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        if (elect_one()) {
            mma_commit(&bar_drain);
            if (!mbar_wait_bounded(&bar_drain, 0, kWaitNs)) report_timeout(a, 10);
        }
        __syncwarp();
    }
    if (tid == 0) {
        for (int cc = max(0, k_issued - 3); cc < k_issued; ++cc)
            if (!mbar_wait_bounded(kbar(cc), kpar(cc), kWaitNs)) report_timeout(a, 11);
        for (int cc = max(0, v_issued - 2); cc < v_issued; ++cc)
            if (!mbar_wait_bounded(&bar_v[cc & 1], (uint32_t)((cc >> 1) & 1), kWaitNs)) report_timeout(a, 11);
    }
    __syncthreads();
    cluster_sync();
    if (!front && tid == 0) {
        const uint32_t issued = ld_shared_cluster_u32(peer_copies);
        for (uint32_t j = s_ops_seen; j < issued; ++j)
            if (!mbar_wait_bounded(&bar_ops[j & 1], (j >> 1) & 1, kWaitNs)) report_timeout(a, 12);
    }
    __syncthreads();
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, front ? 64u : 256u);
    }
}

}  // namespace

cudaError_t launch_replay_pair(const CallArgs& a, cudaStream_t stream) {
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
    const uint32_t smem = PairLayout::BYTES + 1024;
    const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(replay_pair_kernel), (int)smem, smem_set);
    if (e != cudaSuccess) return e;
    replay_pair_kernel<<<(unsigned)(2 * a.units), NT, smem, stream>>>(p, mk, mv);
    return cudaGetLastError();
}

}  // namespace gdn
