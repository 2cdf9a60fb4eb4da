// gdn_replay_ws.cu -- the state-only tail replay on tcgen05 tensor cores with
// warp-specialised roles (bf16 k/v, d_k = d_v = 128, fp32 state in tensor
// memory), one CTA per SM.  Plans run it only when the descriptor pins it
// (GDN_KERNEL_CHUNKED_TC_WARP_SPEC); by default every replay runs the
// two-CTA-per-SM kernel of gdn_replay.cu, which is faster at every launch size.
//
// Tail-Replay ("Tail-Replay: Escaping the Curse of Linear Attention in
// Prefix Caching for Hybrid LLMs", section "Mecanismos Principais", item
// "Reconstrucao de Estado Independente") rebuilds each Gated DeltaNet
// layer's state by replaying only the last R tokens of the matched prefix
// from a zero state:
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T.
// The replay runs 64 tokens at a time in the chunkwise WY / UT form
// (Yang et al., "Parallelizing Linear Transformers with the Delta Rule over
// Sequence Length", 2024, with the gate folded in): A_ij = beta_i
// (gamma_i / gamma_j) k_i.k_j, T = (I + A)^-1, U' = T diag(beta) V,
// U = U' - T diag(beta gamma) K S0, S_C = gamma_C S0 + K^T diag(gamma_C / gamma) U.
//
// Grouping.  With E = diag(gamma_C / gamma), the state S = sigma S~ and the
// scale sigma' after the chunk (sigma gamma_C, or 1 when that falls below
// 2^-40 and S~ is rescaled instead), P = K S~0 and
//   U~ = E U / sigma' = (E T diag(beta) / sigma') V - (sigma / sigma') (E T diag(beta gamma)) P,
//   S~_C = S~0 + K^T U~ .
// Both T operands carry every scale, so U~ comes straight out of the tensor
// core into TMEM in fp32 and the state update reads it from there (tf32, A in
// TMEM): the chain of a chunk is MMAs only, U~ -> state update -> P of the
// next chunk -> U~ of the next chunk.
//
// Roles (416 threads):
//   warps 0-3 and 4-7  two front groups, chunk n on group n % 2: K K^T (MMA),
//                      A, T = (I + A)^-1, the keys in fp32 (K-major for P and
//                      MN-major for the state update, whose tf32 B operand
//                      takes only the 32-byte-atom swizzle) and the two T
//                      operands.  None of it depends on the state, so a group
//                      works up to two chunks ahead of the chain.
//   warps 8-11         the chain: warp 8 issues U~, the state update and P;
//                      all four rescale the state when sigma is folded into it
//                      and write the final state (TMEM lane quarter w % 4 each).
//   warp 12            TMA of the K and V tiles and the gate factors (with the
//                      running sigma) of every chunk.
// Every hand-off is an mbarrier; every wait gives up after 1 s, sets the
// workspace status and makes every role leave its loop.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn_chunk_common.h"

namespace gdn {
namespace {

using namespace sm100;
using namespace chunk;

// Gate factors of one chunk and the scales the chunk's T operands carry.
struct WsGates {
    Gates g;
    float inv_snew;   // 1 / sigma'
    float ratio;      // sigma / sigma'
    float renorm;     // factor folded into S~ before this chunk's update (may be 0), or -1: none
    float snew;       // sigma'
};

constexpr int WS_THREADS = 416;
constexpr int NGATES = 4;   // gate slots, chunk n in n % 4

// ---- shared memory (byte offsets from a 1 KB aligned base) ----
struct WsLayout {
    static constexpr uint32_t BOX = 8192;                   // 64 rows x 64 bf16 (128-byte swizzle)
    static constexpr uint32_t SLOT = 2 * BOX;               // one K or V tile: [d 0-63 | d 64-127]
    static constexpr uint32_t OFF_K = 0;                    // chunk n in slot n % 2
    static constexpr uint32_t OFF_V = OFF_K + 2 * SLOT;     // chunk n in slot n % 2
    // the keys in fp32, [j][dk] in four 8 KB blocks of 32 columns, 128-byte rows:
    // K32P (K-major, 16-byte chunks swizzled, the B operand of P; one buffer, the
    // chunk whose P is next) and K32S (MN-major, 32-byte chunks swizzled, the B
    // operand of the state update; chunk n in n % 2)
    static constexpr uint32_t K32_BYTES = 32768;
    static constexpr uint32_t OFF_K32P = OFF_V + 2 * SLOT;
    static constexpr uint32_t OFF_K32S = OFF_K32P + K32_BYTES;
    // per front group: the bf16 T operand, then A, T and the fp32 T operand in place
    static constexpr uint32_t G_TB = 0;
    static constexpr uint32_t G_AT = 8192;
    static constexpr uint32_t G_BYTES = G_AT + C * LDT * 4;
    static constexpr uint32_t OFF_G = OFF_K32S + 2 * K32_BYTES;
    static constexpr uint32_t OFF_GATES = OFF_G + 2 * G_BYTES;
    static constexpr uint32_t BYTES = OFF_GATES + NGATES * sizeof(WsGates);
};
static_assert(WsLayout::G_BYTES % 1024 == 0, "second group's operands on 1 KB");
static_assert(2 * 8192 <= C * LDT * 4, "the fp32 T operand fits over T");
static_assert(WsLayout::OFF_GATES % 16 == 0, "gate slots aligned");
static_assert(WsLayout::BYTES + 1024 <= 227 * 1024, "fits one CTA's shared memory");

// TMEM columns (512 allocated): S~^T (lane = value row), two 64-column regions
// that alternate between chunks (chunk n's U~ in region n % 2, then P of chunk
// n + 1 over it), and one K K^T region per front group.
constexpr uint32_t TM_STATE = 0;
constexpr uint32_t TM_R0 = 128;
constexpr uint32_t TM_KK0 = 256;

constexpr uint32_t BAR_GRP0 = 1;   // named barriers of the front groups (1, 2)
constexpr uint32_t BAR_CHAIN = 3;  // the chain warps, once at the start

constexpr int MSG_RENORM = 1, MSG_FINISH = 2, MSG_ABORT = 3;

// Wait for an mbarrier phase; false once the CTA aborts or after kWaitNs.
__device__ __forceinline__ bool wait_ab(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                        const CallArgs& a, uint32_t where) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > kWaitNs) {
            report_timeout(a, where);
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

// A of one chunk from its K K^T (M = 64 accumulator, row r in lane 32 (r / 16) +
// r % 16): A = strict_tril(beta_i (gamma_i / gamma_j) K K^T), fp32 into AT, over
// the 32 columns [cb, cb + 32).  This thread takes rows i0 = 16 wq + lane / 4
// and i0 + 8, columns cb + 8 k + 2 (lane % 4) + {0, 1}, k = 0..3.
__device__ __forceinline__ void epilogue_a(uint32_t taddr, const Gates& G, float* AT, int wq, int lane, int cb) {
    const bool fast = G.g2[C - 1] >= kFastGateFloor;
    float v[16];
    tmem_ld16x256b_x4(taddr + cb, v);
    const int i0 = 16 * wq + (lane >> 2), jb = cb + 2 * (lane & 3);
    const float* colf = fast ? G.binv : G.g2;   // column factor: 2^-G_j, or G_j
    float2 cf[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) cf[k] = *reinterpret_cast<const float2*>(colf + jb + 8 * k);
    float gi[2], bi[2], rowf[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int i = i0 + 8 * hf;
        gi[hf] = G.g2[i];
        bi[hf] = G.beta[i];
        rowf[hf] = bi[hf] * G.gam[i];
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
}

// The two T operands of a chunk from T (fp32 in AT), 128 threads (thread ->
// row j = ltid % 64, columns 32 part .. 32 part + 31 with part = ltid / 64):
//   tb : E T diag(beta) / sigma', bf16 [j][j'] in 128-byte swizzled rows;
//   AT : -(sigma / sigma') E T diag(beta gamma), fp32 K-major [j][j'] in two
//        8 KB blocks of 32 columns (128-byte swizzled), over T itself: every
//        thread reads its values, the group meets at barrier `bar`, then writes.
// Consecutive threads take consecutive rows, so the row reads (stride LDT) and
// the swizzled stores are free of bank conflicts.
__device__ __forceinline__ void write_t_operands_grp(float* AT, const WsGates& W, uint8_t* tb, int ltid,
                                                     uint32_t bar) {
    const int j = ltid & (C - 1), part = ltid >> 6;
    const float ej = W.g.e[j];
    const float cb = ej * W.inv_snew;
    const float cg = -W.ratio * ej;
    float vb[32], vg[32];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int col = part * 32 + half * 16 + 4 * q;
            float4 tt = make_float4(0.f, 0.f, 0.f, 0.f);
            if ((col >> 4) <= (j >> 4)) tt = *reinterpret_cast<const float4*>(AT + j * LDT + col);
            const float4 b4 = *reinterpret_cast<const float4*>(W.g.beta + col);
            const float4 g4 = *reinterpret_cast<const float4*>(W.g.gam + col);
            const float tv[4] = {tt.x, tt.y, tt.z, tt.w};
            const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
            const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float tbv = tv[e] * bv[e];
                vb[16 * half + 4 * q + e] = tbv * cb;
                vg[16 * half + 4 * q + e] = tbv * gv[e] * cg;
            }
        }
    }
    named_sync(bar, 128);   // every read of T is done before the fp32 operand overwrites it
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {   // bf16 chunks 4 part + ch of row j
        uint4 x;
        x.x = pack_bf16(vb[ch * 8 + 0], vb[ch * 8 + 1]);
        x.y = pack_bf16(vb[ch * 8 + 2], vb[ch * 8 + 3]);
        x.z = pack_bf16(vb[ch * 8 + 4], vb[ch * 8 + 5]);
        x.w = pack_bf16(vb[ch * 8 + 6], vb[ch * 8 + 7]);
        st_shared_v4(tb, (uint32_t)(j * 128 + (((4 * part + ch) ^ (j & 7)) << 4)), x);
    }
    uint8_t* blk = reinterpret_cast<uint8_t*>(AT) + part * 8192 + j * 128;
#pragma unroll
    for (int q = 0; q < 8; ++q)   // fp32 chunk q of row j in block `part`
        *reinterpret_cast<float4*>(blk + ((q ^ (j & 7)) << 4)) =
            make_float4(vg[4 * q], vg[4 * q + 1], vg[4 * q + 2], vg[4 * q + 3]);
}

// Keys of one chunk (bf16 K slot: two 8 KB boxes of 64 rows x 64 columns,
// 128-byte swizzled) to fp32, [j][dk] in four 8 KB blocks of 32 columns with
// 128-byte rows, twice: k32p with 16-byte chunks swizzled (chunk c of row j at
// c ^ (j % 8); skipped when null) and k32s with 32-byte chunks swizzled (chunk c
// at c ^ (j % 4)).  Rows j >= nrows are written as zeros.  128 threads: thread
// ct -> row j = ct % 64, columns 64 h .. 64 h + 63 with h = ct / 64.
__device__ __forceinline__ void convert_keys_f32(const uint8_t* kslot, uint8_t* k32p, uint8_t* k32s, int ct,
                                                 int nrows) {
    const int j = ct & (C - 1), h = ct >> 6;
    const uint8_t* src = kslot + h * 8192 + j * 128;
    const bool live = j < nrows;
    uint4 raw[8];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch)
        raw[ch] = live ? *reinterpret_cast<const uint4*>(src + ((ch ^ (j & 7)) << 4)) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {   // columns 64 h + 8 ch .. + 7
        const uint32_t wds[4] = {raw[ch].x, raw[ch].y, raw[ch].z, raw[ch].w};
        float f[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            f[2 * e] = __uint_as_float(wds[e] << 16);
            f[2 * e + 1] = __uint_as_float(wds[e] & 0xffff0000u);
        }
        const uint32_t row = (2 * h + (ch >> 2)) * 8192 + j * 128;
        if (k32p) {
            *reinterpret_cast<float4*>(k32p + row + (((2 * (ch & 3)) ^ (j & 7)) << 4)) =
                make_float4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<float4*>(k32p + row + (((2 * (ch & 3) + 1) ^ (j & 7)) << 4)) =
                make_float4(f[4], f[5], f[6], f[7]);
        }
        uint8_t* c32 = k32s + row + (((ch & 3) ^ (j & 3)) << 5);
        *reinterpret_cast<float4*>(c32) = make_float4(f[0], f[1], f[2], f[3]);
        *reinterpret_cast<float4*>(c32 + 16) = make_float4(f[4], f[5], f[6], f[7]);
    }
}

// Rows past the window of a partial chunk's K or V tile to zero (128 threads).
__device__ __forceinline__ void zero_tail(uint8_t* slot, int nrows, int ltid) {
    const int nz = C - nrows;
    for (int e = ltid; e < 2 * nz * 8; e += 128) {
        const int bx = e / (nz * 8), rr = nrows + (e / 8) % nz, ch = e % 8;
        st_shared_v4(slot + bx * WsLayout::BOX, (uint32_t)(rr * 128 + ch * 16), make_uint4(0, 0, 0, 0));
    }
}

// S~ *= s over this warp's TMEM lane quarter (128 columns).
__device__ __forceinline__ void rescale_state_quarter(uint32_t tlane, float s) {
#pragma unroll 1
    for (int cb = 0; cb < 4; ++cb) {
        float sv[32];
        tmem_ld32(tlane + TM_STATE + cb * 32, sv);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) sv[q] *= s;
        tmem_st32(tlane + TM_STATE + cb * 32, sv);
    }
    tmem_wait_st();
}

// S[dk][dv] = s * TMEM[lane dv][dk] for this warp's lanes dv = row.
__device__ __forceinline__ void write_state_quarter(uint32_t tlane, float s, float* out, int row) {
#pragma unroll 1
    for (int cb = 0; cb < 4; ++cb) {
        float v[32];
        tmem_ld32(tlane + TM_STATE + cb * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) out[(size_t)(cb * 32 + i) * D + row] = s * v[i];
    }
}

__global__ void __launch_bounds__(WS_THREADS, 1)
replay_ws_kernel(const TcParams p, const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_v) {
    using L = WsLayout;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // full / free pairs of every ring, the K K^T of each group, the chain's own
    // MMA completions, the chain's messages to warps 9-11, and the final drains
    __shared__ uint64_t bar_k[2], bar_v[2], k_free[2], v_free[2], gfull[NGATES], gfree[NGATES];
    __shared__ uint64_t bar_kk[2], k32p_full, k32p_free[2], k32s_full[2], k32s_free[2], t_full[2], t_free[2];
    __shared__ uint64_t bar_u, bar_s, bar_p, msg_full, msg_ack, bar_fin[3];
    __shared__ uint32_t tmem_slot;
    __shared__ int s_abort;
    __shared__ int s_msg_kind;
    __shared__ float s_msg_scale;

    const CallArgs& a = p.a;
    record_call(a);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3;   // TMEM lane quarter
    const Unit u = a.unit_list[blockIdx.x];
    const int b = u.seq, h = u.head, H = a.num_heads;
    if (!window_agrees(a, b)) {
        if (tid == 0) report_status(a, kStatusMismatch);
        return;
    }
    const Window w = a.windows[b];
    const int nchunks = (w.len + C - 1) / C;
    if (!index_ok(a, b >= 0 && b < a.batch && h >= 0 && h < H && w.row0 >= 0 && w.len >= 0 &&
                            w.row0 + w.len <= a.rows_total))
        return;

    WsGates* gates = reinterpret_cast<WsGates*>(sm + L::OFF_GATES);
    volatile int* abort_flag = &s_abort;
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_k[i], 1);
            mbar_init(&bar_v[i], 1);
            mbar_init(&k_free[i], 1);
            mbar_init(&v_free[i], 1);
            mbar_init(&bar_kk[i], 1);
            mbar_init(&k32p_free[i], 1);
            mbar_init(&k32s_full[i], 1);
            mbar_init(&k32s_free[i], 1);
            mbar_init(&t_full[i], 1);
            mbar_init(&t_free[i], 1);
        }
        for (int i = 0; i < NGATES; ++i) {
            mbar_init(&gfull[i], 1);
            mbar_init(&gfree[i], 2);   // the front group and the chain
        }
        mbar_init(&k32p_full, 1);
        mbar_init(&bar_u, 1);
        mbar_init(&bar_s, 1);
        mbar_init(&bar_p, 1);
        mbar_init(&msg_full, 1);
        mbar_init(&msg_ack, 3);
        for (int i = 0; i < 3; ++i) mbar_init(&bar_fin[i], 1);
        s_abort = 0;
        mbar_fence_init();
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_slot;
    const uint32_t tlane = tbase + ((uint32_t)(wq * 32) << 16);
    auto nrows_of = [&](int n) { return min(C, w.len - n * C); };
    auto region = [](int n) -> uint32_t { return TM_R0 + (uint32_t)(n & 1) * 64u; };

    if (warp == 12) {
        // =============================== producer ===============================
        int issued_k[2] = {-1, -1}, issued_v[2] = {-1, -1};   // last chunk loaded into each slot
        float al[2], be[2];
        auto load_gates = [&](int n) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int jj = lane + 32 * q;
                al[q] = 1.0f;
                be[q] = 0.0f;
                if (n < nchunks && n * C + jj < w.len) {
                    const long long r = w.row0 + (long long)n * C + jj;
                    if (index_ok(a, r < a.rows_total)) {
                        al[q] = a.alpha[r * H + h];
                        be[q] = a.beta[r * H + h];
                    }
                }
            }
        };
        float sigma = 1.0f;
        load_gates(0);
        for (int n = 0; n < nchunks; ++n) {
            const int slot = n & 1, gs = n & (NGATES - 1);
            bool t = true;
            // ---- K tile of chunk n ----
            if (n >= 2) t = wait_ab(&k_free[slot], ((n >> 1) + 1) & 1, abort_flag, a, 40);
            t = __all_sync(0xffffffffu, t);
            if (!t) break;
            if (elect_one()) {
                uint8_t* dst = sm + L::OFF_K + slot * L::SLOT;
                const int r0 = (int)(w.row0 + (long long)n * C);
                mbar_arrive_expect_tx(&bar_k[slot], L::SLOT);
                tma_load_3d(dst, &map_k, &bar_k[slot], 0, h, r0);
                tma_load_3d(dst + L::BOX, &map_k, &bar_k[slot], 64, h, r0);
            }
            __syncwarp();
            issued_k[slot] = n;
            // ---- gate factors of chunk n (lane l: rows l and l + 32) ----
            if (n >= NGATES) t = wait_ab(&gfree[gs], ((n >> 2) + 1) & 1, abort_flag, a, 41);
            t = __all_sync(0xffffffffu, t);
            if (!t) break;
            {
                WsGates& W = gates[gs];
                float lg[2];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    lg[q] = al[q] > 0.0f ? fmaxf(__log2f(al[q]), kLog2Floor) : kLog2Floor;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const float y = __shfl_up_sync(0xffffffffu, lg[q], off);
                        if (lane >= off) lg[q] += y;
                    }
                }
                lg[1] += __shfl_sync(0xffffffffu, lg[0], 31);
                const float g2C = __shfl_sync(0xffffffffu, lg[1], 31);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int jj = lane + 32 * q;
                    W.g.beta[jj] = be[q];
                    W.g.g2[jj] = lg[q];
                    W.g.gam[jj] = exp2f(lg[q]);
                    W.g.binv[jj] = g2C >= kFastGateFloor ? exp2f(-lg[q]) : 0.0f;
                    W.g.e[jj] = exp2f(g2C - lg[q]);
                }
                float snew = sigma * exp2f(g2C);
                float ren = -1.0f;
                if (snew < kRenormBelow) {
                    ren = snew;
                    snew = 1.0f;
                }
                if (lane == 0) {
                    W.inv_snew = 1.0f / snew;
                    W.ratio = sigma / snew;
                    W.renorm = ren;
                    W.snew = snew;
                }
                sigma = snew;
                __syncwarp();
                if (lane == 0) mbar_arrive(&gfull[gs]);
            }
            load_gates(n + 1);
            // ---- V tile of chunk n ----
            if (n >= 2) t = wait_ab(&v_free[slot], ((n >> 1) + 1) & 1, abort_flag, a, 42);
            t = __all_sync(0xffffffffu, t);
            if (!t) break;
            if (elect_one()) {
                uint8_t* dst = sm + L::OFF_V + slot * L::SLOT;
                const int r0 = (int)(w.row0 + (long long)n * C);
                mbar_arrive_expect_tx(&bar_v[slot], L::SLOT);
                tma_load_3d(dst, &map_v, &bar_v[slot], 0, h, r0);
                tma_load_3d(dst + L::BOX, &map_v, &bar_v[slot], 64, h, r0);
            }
            __syncwarp();
            issued_v[slot] = n;
        }
        // every load this warp issued has landed before the CTA leaves
        for (int s = 0; s < 2; ++s) {
            if (issued_k[s] >= 0) mbar_wait_bounded(&bar_k[s], (issued_k[s] >> 1) & 1, kWaitNs);
            if (issued_v[s] >= 0) mbar_wait_bounded(&bar_v[s], (issued_v[s] >> 1) & 1, kWaitNs);
        }
    } else if (warp < 8) {
        // =============================== front groups ===============================
        const int g = warp >> 2, ltid = tid & 127;
        const uint32_t gbar = BAR_GRP0 + (uint32_t)g;
        uint8_t* gbase = sm + L::OFF_G + g * L::G_BYTES;
        float* AT = reinterpret_cast<float*>(gbase + L::G_AT);
        uint8_t* tb = gbase + L::G_TB;
        const uint32_t kk_col = TM_KK0 + 64u * (uint32_t)g;
        const uint32_t id_kk = idesc_bf16(64, 64, false, false);   // K K^T; row r in lane 32 (r/16) + r%16
        int kk_uses = 0;
        for (int n = g; n < nchunks; n += 2) {
            const int slot = n & 1, use = n >> 1, gs = n & (NGATES - 1);
            const int nrows = nrows_of(n);
            uint8_t* kslot = sm + L::OFF_K + slot * L::SLOT;
            bool t = wait_ab(&gfull[gs], (n >> 2) & 1, abort_flag, a, 10) &&
                     wait_ab(&bar_k[slot], use & 1, abort_flag, a, 11);
            if (t && nrows < C) {
                zero_tail(kslot, nrows, ltid);
                fence_proxy_async_smem();
            }
            tc_fence_before();   // the last chunk's reads of this group's K K^T region are done
            if (!named_sync_and(gbar, 128, t)) break;
            // ---- K K^T of chunk n into the group's region ----
            if (warp == 4 * g) {
                tc_fence_after();
                if (elect_one()) {
                    const uint64_t dk0 = smem_desc_sw128(smem_u32(kslot), 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t d = desc_advance(dk0, (kk >> 2) * L::BOX + (kk & 3) * 32);
                        mma_bf16_ss(tbase + kk_col, d, d, id_kk, kk > 0);
                    }
                    mma_commit(&bar_kk[g]);
                }
                __syncwarp();
            }
            // ---- A (fp32 into AT), once the U~ MMAs two chunks back are done with AT's fp32
            //      T operand and with the bf16 one ----
            const WsGates& W = gates[gs];
            t = (n < 2) || wait_ab(&t_free[g], (use + 1) & 1, abort_flag, a, 15);
            t = t && wait_ab(&bar_kk[g], kk_uses & 1, abort_flag, a, 12);
            t = __all_sync(0xffffffffu, t) != 0;   // the TMEM loads below are warp-collective
            ++kk_uses;
            tc_fence_after();
            if (t) {
                epilogue_a(tlane + kk_col, W.g, AT, wq, lane, 0);
                if (wq >= 2) epilogue_a(tlane + kk_col, W.g, AT, wq, lane, 32);
            }
            tc_fence_before();
            if (!named_sync_and(gbar, 128, t)) break;
            // ---- T = (I + A)^-1 in place (scratch in AT's unused upper-right quarter) ----
            invert_unit_lower_inplace<GDN_INV_SCRATCH_IN_AT>(AT, AT + 32, ltid, gbar);
            // ---- the keys in fp32: K32P once P of chunk n - 1 has read it (chunk 0 has no
            //      P), K32S[n % 2] once the state update of chunk n - 2 has ----
            t = (n < 2) || (wait_ab(&k32p_free[g], (use + 1) & 1, abort_flag, a, 13) &&
                            wait_ab(&k32s_free[slot], (use + 1) & 1, abort_flag, a, 16));
            if (t) {
                convert_keys_f32(kslot, n > 0 ? sm + L::OFF_K32P : nullptr, sm + L::OFF_K32S + slot * L::K32_BYTES,
                                 ltid, nrows);
                fence_proxy_async_smem();
            }
            if (!named_sync_and(gbar, 128, t)) break;
            if (ltid == 0) {
                if (n > 0) mbar_arrive(&k32p_full);
                mbar_arrive(&k32s_full[slot]);
                mbar_arrive(&k_free[slot]);   // K K^T and the conversion are done with the tile
            }
            // ---- the T operands ----
            if (nrows < C) {   // the values' rows past the window read as zero
                t = wait_ab(&bar_v[slot], use & 1, abort_flag, a, 14);
                if (t) {
                    zero_tail(sm + L::OFF_V + slot * L::SLOT, nrows, ltid);
                    fence_proxy_async_smem();
                }
                if (!named_sync_and(gbar, 128, t)) break;
            }
            write_t_operands_grp(AT, W, tb, ltid, gbar);
            fence_proxy_async_smem();
            if (!named_sync_and(gbar, 128, true)) break;
            if (ltid == 0) {
                mbar_arrive(&t_full[g]);
                mbar_arrive(&gfree[gs]);
            }
        }
        // the group's own MMAs have completed before the CTA leaves
        if (warp == 4 * g) {
            if (elect_one()) {
                mma_commit(&bar_fin[g]);
                mbar_wait_bounded(&bar_fin[g], 0, kWaitNs);
            }
            __syncwarp();
        }
    } else {
        // =============================== chain ===============================
        {   // zero state
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.0f;
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) tmem_st32(tlane + TM_STATE + cb * 32, v);
            tmem_wait_st();
        }
        tc_fence_before();
        named_sync(BAR_CHAIN, 128);
        tc_fence_after();
        const size_t state_base = ((size_t)b * H + h) * D * D;
        const int row = wq * 32 + lane;   // this thread's TMEM lane: value row dv
        if (warp == 8) {
            const uint32_t id_w = idesc_bf16(128, 64, true, false);    // V^T (E T diag(beta) / sigma')^T
            const uint32_t id_t = idesc_tf32(128, 64, false, false);   // P^T = S~^T K^T, P^T (tbg)^T; A in TMEM
            const uint32_t id_su = idesc_tf32(128, 128, false, true);  // U~^T K, A in TMEM, B (fp32 keys) MN-major
            int nmsg = 0;
            float sigma_fin = 1.0f;
            bool ok = true;
            for (int n = 0; n < nchunks && ok; ++n) {
                const int slot = n & 1, use = n >> 1, gs = n & (NGATES - 1);
                const uint32_t ru = region(n);
                bool t = wait_ab(&gfull[gs], (n >> 2) & 1, abort_flag, a, 20);
                float ren = -1.0f, sn = 1.0f;
                if (t) {
                    ren = gates[gs].renorm;
                    sn = gates[gs].snew;
                }
                __syncwarp();
                if (t && lane == 0) mbar_arrive(&gfree[gs]);
                t = t && wait_ab(&t_full[slot], use & 1, abort_flag, a, 21) &&
                    wait_ab(&bar_v[slot], use & 1, abort_flag, a, 22);
                if (n > 0) t = t && wait_ab(&bar_p, (n - 1) & 1, abort_flag, a, 23);
                if (!__all_sync(0xffffffffu, t)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // ---- U~ of chunk n: V^T (tb)^T, then + P^T (tbg)^T ----
                if (elect_one()) {
                    uint8_t* gb = sm + L::OFF_G + slot * L::G_BYTES;
                    const uint64_t dv = smem_desc_sw128(smem_u32(sm + L::OFF_V + slot * L::SLOT), L::BOX, 1024);
                    const uint64_t dt = smem_desc_sw128(smem_u32(gb + L::G_TB), 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ss(tbase + ru, desc_advance(dv, kk * 2048), desc_advance(dt, kk * 32), id_w,
                                    kk > 0 ? 1u : 0u);
                    if (n > 0) {
                        const uint64_t d2 = smem_desc_sw128(smem_u32(gb + L::G_AT), 16, 1024);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_tf32_ts(tbase + ru, tbase + region(n - 1) + kk * 8,
                                        desc_advance(d2, (kk >> 2) * 8192 + (kk & 3) * 32), id_t, 1u);
                    }
                    mma_commit(&bar_u);
                    mma_commit(&v_free[slot]);
                    mma_commit(&t_free[slot]);
                }
                __syncwarp();
                t = wait_ab(&bar_u, n & 1, abort_flag, a, 24) && wait_ab(&k32s_full[slot], use & 1, abort_flag, a, 25);
                if (!__all_sync(0xffffffffu, t)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // ---- sigma folded into the state (P of chunk n has read it) ----
                if (ren >= 0.0f) {
                    if (lane == 0) {
                        s_msg_kind = MSG_RENORM;
                        s_msg_scale = ren;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&msg_full);
                    rescale_state_quarter(tlane, ren);
                    tc_fence_before();
                    t = wait_ab(&msg_ack, nmsg & 1, abort_flag, a, 26);
                    ++nmsg;
                    if (!__all_sync(0xffffffffu, t)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                // ---- S~^T += U~^T K (K32S: MN-major, 32-byte-atom swizzle, 8 rows per MMA) ----
                if (elect_one()) {
                    const uint64_t dk =
                        smem_desc_sw128_32b(smem_u32(sm + L::OFF_K32S + slot * L::K32_BYTES), 8192, 512);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_tf32_ts(tbase + TM_STATE, tbase + ru + kk * 8, desc_advance(dk, kk * 1024), id_su, 1u);
                    mma_commit(&bar_s);
                    mma_commit(&k32s_free[slot]);
                }
                __syncwarp();
                sigma_fin = sn;
                // ---- P^T of chunk n + 1 = S~^T K_{n+1}^T into region n ----
                if (n + 1 < nchunks) {
                    t = wait_ab(&bar_s, n & 1, abort_flag, a, 27) && wait_ab(&k32p_full, n & 1, abort_flag, a, 28);
                    if (!__all_sync(0xffffffffu, t)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (elect_one()) {
                        const uint64_t dk = smem_desc_sw128(smem_u32(sm + L::OFF_K32P), 16, 1024);
#pragma unroll
                        for (int kk = 0; kk < 16; ++kk)
                            mma_tf32_ts(tbase + ru, tbase + TM_STATE + kk * 8,
                                        desc_advance(dk, (kk >> 2) * 8192 + (kk & 3) * 32), id_t, kk > 0);
                        mma_commit(&bar_p);
                        mma_commit(&k32p_free[n & 1]);   // K32P is free for chunk n + 2
                    }
                    __syncwarp();
                }
            }
            if (ok && nchunks > 0) {   // the last state update
                const bool t = wait_ab(&bar_s, (nchunks - 1) & 1, abort_flag, a, 29);
                ok = __all_sync(0xffffffffu, t) != 0;
                tc_fence_after();
            }
            ok = ok && !*abort_flag;
            const int kind = (ok && a.state_out) ? MSG_FINISH : MSG_ABORT;
            if (lane == 0) {
                s_msg_kind = kind;
                s_msg_scale = sigma_fin;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&msg_full);
            if (kind == MSG_FINISH) write_state_quarter(tlane, sigma_fin, a.state_out + state_base, row);
            tc_fence_before();
            mbar_wait_bounded(&msg_ack, nmsg & 1, kWaitNs);
            if (elect_one()) {
                mma_commit(&bar_fin[2]);
                mbar_wait_bounded(&bar_fin[2], 0, kWaitNs);
            }
            __syncwarp();
        } else {
            // warps 9-11: rescale or write out their lane quarter when warp 8 says so
            for (int m = 0;; ++m) {
                bool t = mbar_wait_bounded(&msg_full, m & 1, kWaitNs);
                if (!__all_sync(0xffffffffu, t)) {
                    if (lane == 0) {
                        report_timeout(a, 30);
                        *abort_flag = 1;
                    }
                    break;
                }
                const int kind = s_msg_kind;
                const float sc = s_msg_scale;
                tc_fence_after();
                if (kind == MSG_RENORM) rescale_state_quarter(tlane, sc);
                else if (kind == MSG_FINISH) write_state_quarter(tlane, sc, a.state_out + state_base, row);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&msg_ack);
                if (kind != MSG_RENORM) break;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

}  // namespace

cudaError_t launch_replay_ws(const CallArgs& a, cudaStream_t stream) {
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
    const uint32_t smem = WsLayout::BYTES + 1024;
    const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(replay_ws_kernel), (int)smem, smem_set);
    if (e != cudaSuccess) return e;
    replay_ws_kernel<<<(unsigned)a.units, WS_THREADS, smem, stream>>>(p, mk, mv);
    return cudaGetLastError();
}

}  // namespace gdn
