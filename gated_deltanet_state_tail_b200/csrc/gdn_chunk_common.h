// gdn_chunk_common.h -- pieces shared by the chunked tensor-core kernels:
// constants of the 64-token chunking, bf16 tile writers, and the
// unit-lower-triangular inverse used by the chunkwise (WY / UT) form.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include <cuda.h>

#include "gdn_internal.h"
#include "gdn_sm100.h"

namespace gdn {

// [rows][H][128] bf16 rows `row_stride` elements apart, viewed as (d, H, rows), box
// 64 x 1 x 64, 128-byte swizzle, rows past `rows` read as zero (defined with the
// chunked prefill).
bool make_tile_map(CUtensorMap* m, const void* base, int H, long long rows, long long row_stride);

namespace chunk {

using namespace sm100;

constexpr int C = 64;        // chunk length
constexpr int D = 128;       // d_k = d_v
constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s per wait
constexpr float kLog2Floor = -115.0f;         // log2 of a zero gate, clamped (2^-115 ~ 2.4e-35)
constexpr int LDT = 68;                       // fp32 row stride of A and T (conflict-free fragments)

constexpr float kRenormBelow = 9.094947e-13f;   // 2^-40: fold sigma into the state below this
constexpr float kFastGateFloor = -100.0f;       // log2 of the chunk decay above which exp2 factorises

__device__ __forceinline__ void st_shared_v4(uint8_t* base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4*>(base + off) = v;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

// Write 32 fp32 values as bf16 into the 16-byte chunks c0 .. c0 + 3
// (columns 8 c0 .. 8 c0 + 31) of the 128-byte swizzled row `row` of the tile
// at `tile`.
__device__ __forceinline__ void write_row32_bf16(uint8_t* tile, int row, int c0, const float* v) {
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        uint4 q;
        q.x = pack_bf16(v[ch * 8 + 0], v[ch * 8 + 1]);
        q.y = pack_bf16(v[ch * 8 + 2], v[ch * 8 + 3]);
        q.z = pack_bf16(v[ch * 8 + 4], v[ch * 8 + 5]);
        q.w = pack_bf16(v[ch * 8 + 6], v[ch * 8 + 7]);
        st_shared_v4(tile, (uint32_t)(row * 128 + (((c0 + ch) ^ (row & 7)) << 4)), q);
    }
}

__device__ __forceinline__ void report_timeout(const CallArgs& a, uint32_t where) {
    report_status(a, kStatusTimeout);
    tag_merge(&a.ws->where, a.epoch, where, true);
}

// acc[nt] += A (16 x 16) * B (16 x 16), nt = two 8-column halves of the result;
// A and B row-major fp32 in shared memory (strides lda, ldb), read as tf32 (the
// tensor core uses the top 19 bits).  With SPLIT_K the two 8-deep k-steps go to
// separate accumulators, summed at the end, so neither product waits for the
// other: a warp-level MMA shares the tensor pipe with the CTA's tcgen05 work and
// its latency grows with it.  That pays where one CTA per SM waits on the
// inverse; with two CTAs per SM the extra instructions cost more than it saves.
template <bool SPLIT_K>
__device__ __forceinline__ void mma16x16_tf32(float acc[2][4], const float* A, int lda, const float* B, int ldb,
                                              int g, int t) {
    auto load_ks = [&](int ks, uint32_t af[4], uint32_t bf[2][2]) {
        af[0] = __float_as_uint(A[g * lda + 8 * ks + t]);
        af[1] = __float_as_uint(A[(g + 8) * lda + 8 * ks + t]);
        af[2] = __float_as_uint(A[g * lda + 8 * ks + t + 4]);
        af[3] = __float_as_uint(A[(g + 8) * lda + 8 * ks + t + 4]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            bf[nt][0] = __float_as_uint(B[(8 * ks + t) * ldb + 8 * nt + g]);
            bf[nt][1] = __float_as_uint(B[(8 * ks + t + 4) * ldb + 8 * nt + g]);
        }
    };
    if (SPLIT_K) {
        float acc1[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        uint32_t af[2][4], bf[2][2][2];
        load_ks(0, af[0], bf[0]);
        load_ks(1, af[1], bf[1]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            mma_sync_tf32(acc[nt], af[0], bf[0][nt]);
            mma_sync_tf32(acc1[nt], af[1], bf[1][nt]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] += acc1[nt][e];
    } else {
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t af[4], bf[2][2];
            load_ks(ks, af, bf);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) mma_sync_tf32(acc[nt], af, bf[nt]);
        }
    }
}

// Store a 16 x 16 fragment pair (times `scale`) row-major at D (stride ldd).  WIDE:
// one 8-byte store per pair of values (ldd even, D 8-byte aligned), which a warp
// issues as 256 bytes in the minimum two wavefronts, where two 4-byte stores each
// conflict two ways; it keeps both values live, which a kernel at its register cap
// pays for in spills.
template <bool WIDE>
__device__ __forceinline__ void store16x16(float* D, int ldd, const float acc[2][4], float scale, int g, int t) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        if (WIDE) {
            *reinterpret_cast<float2*>(D + g * ldd + 8 * nt + 2 * t) =
                make_float2(scale * acc[nt][0], scale * acc[nt][1]);
            *reinterpret_cast<float2*>(D + (g + 8) * ldd + 8 * nt + 2 * t) =
                make_float2(scale * acc[nt][2], scale * acc[nt][3]);
        } else {
            D[g * ldd + 8 * nt + 2 * t] = scale * acc[nt][0];
            D[g * ldd + 8 * nt + 2 * t + 1] = scale * acc[nt][1];
            D[(g + 8) * ldd + 8 * nt + 2 * t] = scale * acc[nt][2];
            D[(g + 8) * ldd + 8 * nt + 2 * t + 1] = scale * acc[nt][3];
        }
    }
}

// In place: on entry AT (fp32, 64 x LDT) holds the strictly lower triangular
// A (entries on and above the diagonal are ignored); on exit it holds
// T = (I + A)^-1 on and below the diagonal 16 x 16 blocks (the upper
// triangles of the diagonal blocks are written as zeros; the blocks above
// them are left untouched and must be read as zero).  Xs holds the merges'
// four 16 x 16 scratch blocks: block s at Xs + (s / 2) XHI + (s % 2) XLO, row
// stride LDX (see GDN_INV_SCRATCH_IN_AT below).
//
// Diagonal blocks: forward substitution on CUDA cores, warp w solves block w
// with one lane per column.  Then recursive doubling with
// warp-level tf32 tensor-core products: 32 x 32 blocks T_10 = -D_1 A_10 D_0
// and T_32 = -D_3 A_32 D_2 (warps 0-1, while warps 2-3 form the parts of
// X = A_21 T_11 that need only diagonal blocks), then the lower-left 32 x 32
// block -T_22 X (warp (r, c) computes 16 x 16 block (r, c)).  ltid is the
// thread's index among the 128 threads that run it; bar_id names the barrier
// those threads share.
//
// emit sees each 16 x 16 block of T once it is final: emit.prepare() runs on
// all 128 threads after the diagonal solves, before any other emit call (a
// caller whose output buffers are still being read waits there);
// emit.diagonal(AT, q) runs on 64 threads (q = 0..63, warps 0-1, while warps
// 2-3 merge) once the four diagonal blocks are in AT (zeros above their
// diagonals); emit.block(r0, c0, acc, scale, g, t) gets block (r0 / 16, c0 / 16)
// below the diagonal from the registers of the warp that computed it, as scale
// times an m16n8 fragment pair (T[r0 + g + 8 h][c0 + 8 nt + 2 t + e] = scale *
// acc[nt][2 h + e]).
struct NoEmit {
    __device__ __forceinline__ void prepare() const {}
    __device__ __forceinline__ void diagonal(const float*, int) const {}
    __device__ __forceinline__ void block(int, int, const float (&)[2][4], float, int, int) const {}
};

// SPLIT_K selects the variant for a kernel with registers to spare (one CTA per
// SM): the products' k-steps in separate accumulators and 8-byte fragment stores.
template <int LDX, int XHI, int XLO, class Emit = NoEmit, bool SPLIT_K = false>
__device__ __forceinline__ void invert_unit_lower_inplace(float* AT, float* Xs, int ltid, uint32_t bar_id,
                                                          const Emit& emit = Emit()) {
    const int warp = ltid >> 5, lane = ltid & 31;
    // scratch block s (16 x 16, row stride LDX) of the merges
    auto xslot = [&](int s) { return Xs + (s >> 1) * XHI + (s & 1) * XLO; };
    {
        // every lane computes; lanes 16..31 repeat lanes 0..15 and do not store.
        // Row i of the block is read four entries per (broadcast) load.
        const int o = warp * 16, cc = lane & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float s0 = (i == cc) ? 1.0f : 0.0f, s1 = 0.0f;
#pragma unroll
            for (int j4 = 0; j4 < i; j4 += 4) {
                const float4 a4 = *reinterpret_cast<const float4*>(AT + (o + i) * LDT + o + j4);
                const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = j4 + e;
                    if (j < i) {
                        if (j & 1) s1 = fmaf(-av[e], x[j], s1);
                        else s0 = fmaf(-av[e], x[j], s0);
                    }
                }
            }
            x[i] = s0 + s1;
        }
        __syncwarp();
        if (lane < 16) {
#pragma unroll
            for (int i = 0; i < 16; ++i) AT[(o + i) * LDT + o + cc] = x[i];
        }
    }
    named_sync(bar_id, 128);
    emit.prepare();
    const int g = lane >> 2, t = lane & 3;
    // Level A, warps 0-1: 32 x 32 merges, warp 0 -> block (1, 0), warp 1 -> block (3, 2),
    // T_ba = -D_b (A_ba D_a).  Warps 2-3 meanwhile start block row r = warp of the
    // lower-left X = A_21 T_11 from the diagonal blocks alone: P_r0 = A_r0 D_0 and
    // X_r1 = A_r1 D_1 (kept in registers).
    float pr0[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float xr1[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    if (warp < 2) {
        float* X = xslot(warp);
        const int bo = warp ? 48 : 16, ao = warp ? 32 : 0;   // row block b, column block a
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        mma16x16_tf32<SPLIT_K>(acc, AT + bo * LDT + ao, LDT, AT + ao * LDT + ao, LDT, g, t);     // A_ba D_a
        store16x16<SPLIT_K>(X, LDX, acc, 1.0f, g, t);
        __syncwarp();
        float r[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        mma16x16_tf32<SPLIT_K>(r, AT + bo * LDT + bo, LDT, X, LDX, g, t);                      // D_b (A_ba D_a)
        store16x16<SPLIT_K>(AT + bo * LDT + ao, LDT, r, -1.0f, g, t);
        emit.block(bo, ao, r, -1.0f, g, t);
    } else {
        const int r = warp;
        mma16x16_tf32<SPLIT_K>(pr0, AT + 16 * r * LDT, LDT, AT, LDT, g, t);                    // A_r0 D_0
        mma16x16_tf32<SPLIT_K>(xr1, AT + 16 * r * LDT + 16, LDT, AT + 16 * LDT + 16, LDT, g, t);  // A_r1 D_1
    }
    named_sync(bar_id, 128);
    // Level B: X_r0 = P_r0 + A_r1 T_10 (warps 2-3), X blocks to the scratch, slot 2 (r - 2) + c
    if (warp >= 2) {
        const int r = warp;
        mma16x16_tf32<SPLIT_K>(pr0, AT + 16 * r * LDT + 16, LDT, AT + 16 * LDT, LDT, g, t);      // + A_r1 T_10
        store16x16<SPLIT_K>(xslot(2 * (r - 2)), LDX, pr0, 1.0f, g, t);
        store16x16<SPLIT_K>(xslot(2 * (r - 2) + 1), LDX, xr1, 1.0f, g, t);
    } else {
        emit.diagonal(AT, ltid);
    }
    named_sync(bar_id, 128);    // X blocks visible; every read of A_21 done
    // then T_21 = -T_22 X, warp w -> block (r, c) = (2 + w / 2, w % 2)
    {
        const int r = 2 + (warp >> 1), c = warp & 1;
        float rr[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const float* X2c = xslot(c);
        if (r == 2) {
            mma16x16_tf32<SPLIT_K>(rr, AT + 32 * LDT + 32, LDT, X2c, LDX, g, t);              // D_2 X_2c
        } else {
            const float* X3c = xslot(2 + c);
            mma16x16_tf32<SPLIT_K>(rr, AT + 48 * LDT + 32, LDT, X2c, LDX, g, t);              // T_32 X_2c
            mma16x16_tf32<SPLIT_K>(rr, AT + 48 * LDT + 48, LDT, X3c, LDX, g, t);              // D_3 X_3c
        }
        store16x16<SPLIT_K>(AT + 16 * r * LDT + 16 * c, LDT, rr, -1.0f, g, t);
        emit.block(16 * r, 16 * c, rr, -1.0f, g, t);
    }
    named_sync(bar_id, 128);
}

// The inverse's scratch placement: the upper-right 32 x 32 quarter of AT itself
// (rows 0-31, columns 32-63), which neither A nor T uses; pass AT + 32 as Xs.
#define GDN_INV_SCRATCH_IN_AT LDT, 16 * LDT, 16

// ---------------------------------------------------------------- kernel building blocks
// Shared by the replay and prefill kernels of the chunked tensor-core path.

constexpr int NT = 256;      // threads per CTA

// ---- the prefill's tile slot (byte offsets inside a slot of 48 KB) ----
// Two slots (chunk c in slot c % 2, the next chunk prefetched by TMA), made of
// 8 KB boxes of 64 rows x 64 columns: [K0 | Q0 | K1 | Q1 | V0 | V1], the K block
// stride 16 KB so that [K; Q] is one 128-row operand.  (The replay keeps its own
// map in gdn_replay.cu.)
struct TileLayout {
    static constexpr uint32_t TILE = 49152;
    static constexpr uint32_t K_BLK = 16384;   // stride of the two K blocks
    static constexpr uint32_t Q0 = 8192;
    static constexpr uint32_t V0 = 32768;
    static constexpr uint32_t V_LBO = 8192;
};

// TMEM columns (the state in both kernels; the rest is the prefill's map, the
// replay keeps its own regions in gdn_replay.cu)
constexpr uint32_t TM_S = 0;      // 128 columns: fp32 S^T / sigma, lane = value row, column = key
constexpr uint32_t TM_U = 128;    // 64 columns: U'^T then U^T, lane = value row
constexpr uint32_t TM_P = 192;    // 64 columns: [K;Q] K^T, then W^T (lane = key)
constexpr uint32_t TM_O = 256;    // 64 columns (prefill): O^T, lane = value row
constexpr uint32_t TM_UB = 320;   // 32 columns (prefill): U^T in bf16, two chunk rows per column
constexpr uint32_t TM_UT = 352;   // 32 columns (prefill): U~^T = U^T diag(e) / sigma in bf16

struct TcParams {
    CallArgs a;
};

// Per-chunk gate factors: beta, G = cumulative log2 decay, gamma = 2^G,
// binv = 2^-G (when the chunk's total decay is >= 2^-100), e = 2^(G_C - G).
struct Gates {
    alignas(16) float beta[C];
    alignas(16) float g2[C];
    alignas(16) float gam[C];
    alignas(16) float binv[C];
    alignas(16) float e[C];
    float scan;
};

constexpr uint32_t BAR_GATES = 3;   // named barrier of warps 0-1
constexpr uint32_t BAR_INV = 1;     // named barrier of warps 0-3 (the UT inverse)

// Build the gate factors of one chunk from the fp32 gates of token `tid`
// (identity transitions past the window).  Called by threads 0..63 only
// (warps 0 and 1, which share a named barrier).
__device__ __forceinline__ void build_gates(Gates& G, float al, float be, int tid, int lane) {
    {
        float lg = al > 0.0f ? fmaxf(__log2f(al), kLog2Floor) : kLog2Floor;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            float y = __shfl_up_sync(0xffffffffu, lg, off);
            if (lane >= off) lg += y;
        }
        if (tid == 31) G.scan = lg;
        G.beta[tid] = be;
        G.g2[tid] = lg;
    }
    named_sync(BAR_GATES, 64);
    if (tid >= 32) G.g2[tid] += G.scan;
    named_sync(BAR_GATES, 64);
    {
        const float g2C = G.g2[C - 1];
        const float gj = G.g2[tid];
        G.gam[tid] = exp2f(gj);
        G.binv[tid] = g2C >= kFastGateFloor ? exp2f(-gj) : 0.0f;
        G.e[tid] = exp2f(g2C - gj);
    }
}

// An emitter for invert_unit_lower_inplace: each final block of T goes from
// registers (or, for the diagonal blocks, from AT) into the chunk's two T
// operands,
//   tb[j][j'] = r_j T[j][j'] beta_j'                  (bf16, 128-byte swizzled rows),
//   tg[j][j'] = -sigma' r_j T[j][j'] beta_j' gamma_j' (fp32, K-major, two 8 KB blocks
//                                                      of 32 columns, 128-byte swizzled),
// with r_j = gamma_C / gamma_j (ROW_E, the replay's chunk decay folded into the
// rows) or 1 (the prefill, whose outputs need U itself), and sigma' the state's
// scale entering the chunk.  tg follows tb at tb + 8192.
template <bool ROW_E>
struct TOperandEmit {
    const Gates* G;
    float nsig;    // -sigma'
    uint8_t* tb;   // tg follows at tb + 8192
    uint64_t* bar_rd;    // null, or the mbarrier of the MMAs still reading tb and tg
    uint32_t parity;
    const CallArgs* a;
    int* abort_flag;
    __device__ __forceinline__ void prepare() const {
        if (bar_rd != nullptr && !mbar_wait_bounded(bar_rd, parity, kWaitNs)) {
            report_timeout(*a, 8);
            *abort_flag = 1;
        }
    }
    __device__ __forceinline__ static uint32_t off_b(int j, int jj) {
        return (uint32_t)(j * 128 + (((jj >> 3) ^ (j & 7)) << 4) + (jj & 7) * 2);
    }
    __device__ __forceinline__ static uint32_t off_g(int j, int jj) {
        return (uint32_t)(8192 + (jj >> 5) * 8192 + j * 128 + ((((jj & 31) >> 2) ^ (j & 7)) << 4) + (jj & 3) * 4);
    }
    // thread q: row j = 16 (q / 16) + q % 16 of its diagonal block, 16 columns
    __device__ __forceinline__ void diagonal(const float* AT, int q) const {
        const int o = (q >> 4) * 16, j = o + (q & 15);
        const float ej = ROW_E ? G->e[j] : 1.0f, ejg = nsig * ej;
        float v[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float4 t4 = *reinterpret_cast<const float4*>(AT + j * LDT + o + 4 * k);
            const float4 b4 = *reinterpret_cast<const float4*>(G->beta + o + 4 * k);
            const float4 g4 = *reinterpret_cast<const float4*>(G->gam + o + 4 * k);
            v[4 * k + 0] = t4.x * b4.x;
            v[4 * k + 1] = t4.y * b4.y;
            v[4 * k + 2] = t4.z * b4.z;
            v[4 * k + 3] = t4.w * b4.w;
            const float4 w4 = make_float4(v[4 * k] * g4.x * ejg, v[4 * k + 1] * g4.y * ejg,
                                          v[4 * k + 2] * g4.z * ejg, v[4 * k + 3] * g4.w * ejg);
            *reinterpret_cast<float4*>(tb + off_g(j, o + 4 * k)) = w4;
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint4 x;
            x.x = pack_bf16(v[8 * hh + 0] * ej, v[8 * hh + 1] * ej);
            x.y = pack_bf16(v[8 * hh + 2] * ej, v[8 * hh + 3] * ej);
            x.z = pack_bf16(v[8 * hh + 4] * ej, v[8 * hh + 5] * ej);
            x.w = pack_bf16(v[8 * hh + 6] * ej, v[8 * hh + 7] * ej);
            st_shared_v4(tb, off_b(j, o + 8 * hh), x);
        }
    }
    __device__ __forceinline__ void block(int r0, int c0, const float (&acc)[2][4], float scale, int g,
                                          int t) const {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int jj = c0 + 8 * nt + 2 * t;
            const float2 b2 = *reinterpret_cast<const float2*>(G->beta + jj);
            const float2 g2 = *reinterpret_cast<const float2*>(G->gam + jj);
            const float bg0 = nsig * b2.x * g2.x, bg1 = nsig * b2.y * g2.y;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int j = r0 + g + 8 * hh;
                const float ej = ROW_E ? scale * G->e[j] : scale;
                const float v0 = acc[nt][2 * hh] * ej, v1 = acc[nt][2 * hh + 1] * ej;
                *reinterpret_cast<uint32_t*>(tb + off_b(j, jj)) = pack_bf16(v0 * b2.x, v1 * b2.y);
                *reinterpret_cast<float2*>(tb + off_g(j, jj)) = make_float2(v0 * bg0, v1 * bg1);
            }
        }
    }
};

// Block-wide agreement after a bounded wait: every thread leaves together.
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, const CallArgs& a, uint32_t where) {
    bool ok = mbar_wait_bounded(bar, parity, kWaitNs);
    ok = __syncthreads_and(ok) != 0;
    if (!ok && threadIdx.x == 0) report_timeout(a, where);
    return ok;
}

// TMA of one prefill chunk's tiles: K and V, and Q when the chunk writes outputs.
// (Tile loads need no bounds check: TMA reads zeros past the map's extent.)
__device__ __forceinline__ void issue_tiles(uint8_t* tile, uint64_t* bar, const CUtensorMap* mk, const CUtensorMap* mv,
                                            const CUtensorMap* mq, int h, int r0, bool with_q) {
    using L = TileLayout;
    mbar_arrive_expect_tx(bar, with_q ? L::TILE : 32768u);
    tma_load_3d(tile, mk, bar, 0, h, r0);
    tma_load_3d(tile + L::K_BLK, mk, bar, 64, h, r0);
    tma_load_3d(tile + L::V0, mv, bar, 0, h, r0);
    tma_load_3d(tile + L::V0 + L::V_LBO, mv, bar, 64, h, r0);
    if (with_q) {
        tma_load_3d(tile + L::Q0, mq, bar, 0, h, r0);
        tma_load_3d(tile + L::Q0 + 16384, mq, bar, 64, h, r0);
    }
}

}  // namespace chunk
}  // namespace gdn
