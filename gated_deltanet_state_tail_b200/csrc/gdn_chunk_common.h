// gdn_chunk_common.h -- pieces shared by the chunked tensor-core kernels:
// constants of the 64-token chunking, bf16 tile writers, and the
// unit-lower-triangular inverse used by the chunkwise (WY / UT) form.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "gdn_internal.h"
#include "gdn_sm100.h"

namespace gdn {
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

__device__ __forceinline__ void report_timeout(const CallArgs& a, uint32_t where) {
    atomicOr(&a.ws->status, kStatusTimeout);
    atomicCAS(&a.ws->timeout_where, 0u, where);
}

// In place: on entry AT (fp32, 64 x LDT) holds the strictly lower triangular
// A (entries on and above the diagonal are ignored); on exit it holds
// T = (I + A)^-1 on and below the diagonal 16 x 16 blocks (the upper
// triangles of the diagonal blocks are written as zeros; the blocks above
// them are left untouched and must be read as zero).
//
// The 16 x 16 diagonal blocks are inverted by forward substitution on CUDA
// cores, one lane per column, right-looking (once x_j is final it is pushed
// into the rows below, so the serial dependency is one FMA per row).  The
// blocks below the diagonal follow from T_ba = -T_bb sum_{a <= m < b} A_bm
// T_ma, one block row b at a time, as warp-level tf32 tensor-core products
// (warp a computes block (b, a); the tensor core reads the top 19 bits of
// the fp32 values).  ltid is the thread's index among the 128 threads that
// run it; bar_id names the barrier those threads share.
__device__ __forceinline__ void invert_unit_lower_inplace(float* AT, float* Xs, int ltid, uint32_t bar_id) {
    const int warp = ltid >> 5, lane = ltid & 31;
    {
        // every lane computes; lanes 16..31 repeat lanes 0..15 and do not store
        const int o = warp * 16, cc = lane & 15;
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = (i == cc) ? 1.0f : 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float xj = acc[j];
#pragma unroll
            for (int i = j + 1; i < 16; ++i) acc[i] = fmaf(-AT[(o + i) * LDT + o + j], xj, acc[i]);
        }
        __syncwarp();
        if (lane < 16) {
#pragma unroll
            for (int i = 0; i < 16; ++i) AT[(o + i) * LDT + o + cc] = acc[i];
        }
    }
    named_sync(bar_id, 128);
    const int g = lane >> 2, t = lane & 3;
    for (int b = 1; b < 4; ++b) {
        float* X = Xs + warp * (16 * 24);
        if (warp < b) {
            const int a = warp;
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            for (int m = a; m < b; ++m) {
                uint32_t af[2][4], bf[2][2][2];
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    const int k0 = 16 * m + 8 * ks;
                    af[ks][0] = __float_as_uint(AT[(16 * b + g) * LDT + k0 + t]);
                    af[ks][1] = __float_as_uint(AT[(16 * b + g + 8) * LDT + k0 + t]);
                    af[ks][2] = __float_as_uint(AT[(16 * b + g) * LDT + k0 + t + 4]);
                    af[ks][3] = __float_as_uint(AT[(16 * b + g + 8) * LDT + k0 + t + 4]);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        bf[ks][nt][0] = __float_as_uint(AT[(k0 + t) * LDT + 16 * a + 8 * nt + g]);
                        bf[ks][nt][1] = __float_as_uint(AT[(k0 + t + 4) * LDT + 16 * a + 8 * nt + g]);
                    }
                }
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) mma_sync_tf32(acc[nt], af[ks], bf[ks][nt]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                X[g * 24 + 8 * nt + 2 * t] = acc[nt][0];
                X[g * 24 + 8 * nt + 2 * t + 1] = acc[nt][1];
                X[(g + 8) * 24 + 8 * nt + 2 * t] = acc[nt][2];
                X[(g + 8) * 24 + 8 * nt + 2 * t + 1] = acc[nt][3];
            }
        }
        named_sync(bar_id, 128);   // every read of A_b* is done before T_b* overwrites it
        if (warp < b) {
            const int a = warp;
            uint32_t af[2][4], bf[2][2][2];
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                const int k0 = 8 * ks;
                af[ks][0] = __float_as_uint(AT[(16 * b + g) * LDT + 16 * b + k0 + t]);
                af[ks][1] = __float_as_uint(AT[(16 * b + g + 8) * LDT + 16 * b + k0 + t]);
                af[ks][2] = __float_as_uint(AT[(16 * b + g) * LDT + 16 * b + k0 + t + 4]);
                af[ks][3] = __float_as_uint(AT[(16 * b + g + 8) * LDT + 16 * b + k0 + t + 4]);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    bf[ks][nt][0] = __float_as_uint(X[(k0 + t) * 24 + 8 * nt + g]);
                    bf[ks][nt][1] = __float_as_uint(X[(k0 + t + 4) * 24 + 8 * nt + g]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                float r[4] = {0.f, 0.f, 0.f, 0.f};
                mma_sync_tf32(r, af[0], bf[0][nt]);
                mma_sync_tf32(r, af[1], bf[1][nt]);
                AT[(16 * b + g) * LDT + 16 * a + 8 * nt + 2 * t] = -r[0];
                AT[(16 * b + g) * LDT + 16 * a + 8 * nt + 2 * t + 1] = -r[1];
                AT[(16 * b + g + 8) * LDT + 16 * a + 8 * nt + 2 * t] = -r[2];
                AT[(16 * b + g + 8) * LDT + 16 * a + 8 * nt + 2 * t + 1] = -r[3];
            }
        }
        named_sync(bar_id, 128);
    }
}

// From the inverse T (in place in AT, see above) write the bf16 operands
// T diag(beta) -> tb and T diag(beta gamma) -> tbg, [j][j'] in 128-byte
// swizzled rows.  tb / tbg may overlap AT: every thread reads its values
// before the barrier and writes after it.
__device__ __forceinline__ void write_scaled_t(const float* AT, const float* beta, const float* gam,
                                               uint8_t* tb, uint8_t* tbg, int ltid, uint32_t bar_id) {
    const int j = ltid >> 1, half = ltid & 1;
    float vb[32], vbg[32];
#pragma unroll
    for (int q = 0; q < 32; q += 4) {
        const int col = half * 32 + q;
        float4 tt = make_float4(0.f, 0.f, 0.f, 0.f);
        if ((col >> 4) <= (j >> 4)) tt = *reinterpret_cast<const float4*>(AT + j * LDT + col);
        const float tv[4] = {tt.x, tt.y, tt.z, tt.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x = tv[e] * beta[col + e];
            vb[q + e] = x;
            vbg[q + e] = x * gam[col + e];
        }
    }
    named_sync(bar_id, 128);
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
        st_shared_v4(tb, off, x);
        st_shared_v4(tbg, off, y);
    }
}

}  // namespace chunk
}  // namespace gdn
