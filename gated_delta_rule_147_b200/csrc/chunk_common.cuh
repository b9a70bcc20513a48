// Pieces shared by the chunkwise tensor-core kernels: sizes, launch
// parameters, and bf16 packing helpers for 128-byte-swizzled tiles.
#pragma once

#include "common.cuh"

namespace gdr {
namespace chunkc {

constexpr int C = 64;     // chunk length
constexpr int DK = 128;   // key dimension
constexpr int NV = 64;    // value columns per CTA
constexpr int NT = 256;   // threads per CTA (two warpgroups)

struct Params {
    const void *q, *k, *v;  // raw inputs (for chunks that take the exact path)
    const void* alpha;  // scalar gates are read with plain loads
    const void* bg;
    const void* wg;
    const float* S0;
    __nv_bfloat16* o;
    float* ST;
    int* d_status;
    int B, T, H, dv;
    int akind, bkind, wkind;
    int group;  // value heads per q/k head: q, k have H / group heads, read at h / group
};

__device__ __forceinline__ void st_chunk(uint8_t* base, uint32_t off, const float* x8) {
    uint4 u;
    u.x = pack_bf16x2(x8[0], x8[1]);
    u.y = pack_bf16x2(x8[2], x8[3]);
    u.z = pack_bf16x2(x8[4], x8[5]);
    u.w = pack_bf16x2(x8[6], x8[7]);
    *reinterpret_cast<uint4*>(base + off) = u;
}

__device__ __forceinline__ void st_zero_chunk(uint8_t* base, uint32_t off) {
    *reinterpret_cast<uint4*>(base + off) = make_uint4(0u, 0u, 0u, 0u);
}

// Four bf16 channels [4 cg, 4 cg + 4) of row r of a swizzled 128-column tile.
__device__ __forceinline__ uint32_t piece4(int r, int cg, int rows) {
    return sw128_chunk(r, cg >> 1, rows) + (uint32_t)(cg & 1) * 8u;
}

__device__ __forceinline__ void ld4(const uint8_t* base, uint32_t off, float* x4) {
    const uint2 u = *reinterpret_cast<const uint2*>(base + off);
    const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    x4[0] = f0.x; x4[1] = f0.y; x4[2] = f1.x; x4[3] = f1.y;
}

__device__ __forceinline__ void st4(uint8_t* base, uint32_t off, const float* x4) {
    uint2 u;
    u.x = pack_bf16x2(x4[0], x4[1]);
    u.y = pack_bf16x2(x4[2], x4[3]);
    *reinterpret_cast<uint2*>(base + off) = u;
}

// fp32 [64 x 64] scratch with rows of 16 float4 groups XOR-swizzled by row.
__device__ __forceinline__ float* f32_at(float* base, int r, int c) {
    return base + r * 64 + ((((c >> 2) ^ (r & 15))) << 2) + (c & 3);
}

__device__ __forceinline__ void ld_chunk(const uint8_t* base, uint32_t off, float* x8) {
    uint4 u = *reinterpret_cast<const uint4*>(base + off);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        x8[2 * i] = f.x;
        x8[2 * i + 1] = f.y;
    }
}

// T = (I + A)^-1 for the strictly lower 64 x 64 matrix A (fp32, swizzled rows,
// with its 16 x 16 diagonal blocks also stored transposed at scr[I * 272 +
// j * 16 + rr]) into T32: right-looking forward substitution on the diagonal
// blocks, then recursive halving 16 -> 32 -> 64 on warp-level tensor cores.
// Called by all 256 threads; ends with a block barrier.
__device__ __forceinline__ void solve_unit_lower(float* A32, float* T32, float* scr, int tid, int warp) {
    if (tid < 64) {
        // diagonal block I, column c: right-looking substitution; column j
        // of the block is a contiguous row of the transposed copy AT
        const int I = tid >> 4, c = tid & 15;
        const float* at = scr + I * 272;
        float acc[16], x[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) acc[rr] = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            x[j] = ((j == c) ? 1.f : 0.f) - acc[j];
            float a[16];
#pragma unroll
            for (int r4 = 0; r4 < 16; r4 += 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(at + j * 16 + r4);
                a[r4] = v4.x; a[r4 + 1] = v4.y; a[r4 + 2] = v4.z; a[r4 + 3] = v4.w;
            }
#pragma unroll
            for (int rr = j + 1; rr < 16; ++rr) acc[rr] += a[rr] * x[j];
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) *f32_at(T32, 16 * I + rr, 16 * I + c) = x[rr];
    } else if (tid < 128) {
        // the strictly upper 16x16 blocks inside each 32x32 diagonal half are zero
        const int u = tid - 64;                        // 64 threads, 2 blocks x 16 rows x 4 float4
        for (int idx = u; idx < 128; idx += 64) {
            const int blk = idx >> 6, rr = (idx >> 2) & 15, c4 = (idx & 3) * 4;
            *reinterpret_cast<float4*>(f32_at(T32, 32 * blk + rr, 32 * blk + 16 + c4)) =
                make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    __syncthreads();
    // Merges on warp-level tensor cores (tf32 operands, fp32 accumulate).
    // One warp computes a 16 x 8 tile
    //   D[i][j] = sum_k A[rA + i][cA + k] B[rB + k][cB + j],  k < 8 ksteps,
    // reading A and B from the swizzled fp32 tiles (f32_at) or from a
    // plain scratch tile with rows of kPad floats.
    constexpr int kPad = 40;
    const int lane = tid & 31, gq = lane >> 2, tq = lane & 3;
    auto tile_mma = [&](float* Am, bool swzA, int rA, int cA, float* Bm, bool swzB, int rB,
                        int cB, int ksteps, float* acc) {
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] = 0.f;
        auto ldA = [&](int r, int c) { return swzA ? *f32_at(Am, r, c) : Am[r * kPad + c]; };
        auto ldB = [&](int r, int c) { return swzB ? *f32_at(Bm, r, c) : Bm[r * kPad + c]; };
        for (int ks = 0; ks < ksteps; ++ks) {
            const int k = 8 * ks;
            uint32_t a[4], b[2];
            a[0] = to_tf32(ldA(rA + gq, cA + k + tq));
            a[1] = to_tf32(ldA(rA + gq + 8, cA + k + tq));
            a[2] = to_tf32(ldA(rA + gq, cA + k + tq + 4));
            a[3] = to_tf32(ldA(rA + gq + 8, cA + k + tq + 4));
            b[0] = to_tf32(ldB(rB + k + tq, cB + gq));
            b[1] = to_tf32(ldB(rB + k + tq + 4, cB + gq));
            mma_tf32_m16n8k8(acc, a, b);
        }
    };
    float* XY = scr;  // X: [2][16 x kPad], later Y: [32 x kPad]
    // 16 -> 32: X_b = A_(2b+1)(2b) T_(2b)(2b) (b = 0, 1), four 16 x 8 tiles
    if (warp < 4) {
        const int b = warp >> 1, nt = warp & 1;
        const int R = 32 * b + 16, Cc = 32 * b;
        float acc[4];
        tile_mma(A32, true, R, Cc, T32, true, Cc, Cc + 8 * nt, 2, acc);
        float* X = XY + b * 16 * kPad;
        X[gq * kPad + 8 * nt + 2 * tq] = acc[0];
        X[gq * kPad + 8 * nt + 2 * tq + 1] = acc[1];
        X[(gq + 8) * kPad + 8 * nt + 2 * tq] = acc[2];
        X[(gq + 8) * kPad + 8 * nt + 2 * tq + 1] = acc[3];
    }
    __syncthreads();
    // T_(2b+1)(2b) = -T_(2b+1)(2b+1) X_b
    if (warp < 4) {
        const int b = warp >> 1, nt = warp & 1;
        const int R = 32 * b + 16, Cc = 32 * b;
        float acc[4];
        tile_mma(T32, true, R, R, XY + b * 16 * kPad, false, 0, 8 * nt, 2, acc);
        *f32_at(T32, R + gq, Cc + 8 * nt + 2 * tq) = -acc[0];
        *f32_at(T32, R + gq, Cc + 8 * nt + 2 * tq + 1) = -acc[1];
        *f32_at(T32, R + gq + 8, Cc + 8 * nt + 2 * tq) = -acc[2];
        *f32_at(T32, R + gq + 8, Cc + 8 * nt + 2 * tq + 1) = -acc[3];
    }
    __syncthreads();
    // 32 -> 64: Y = A[32:64, 0:32] T[0:32, 0:32], eight 16 x 8 tiles (one per warp)
    {
        const int mt = warp >> 2, nt = warp & 3;
        float acc[4];
        tile_mma(A32, true, 32 + 16 * mt, 0, T32, true, 0, 8 * nt, 4, acc);
        XY[(16 * mt + gq) * kPad + 8 * nt + 2 * tq] = acc[0];
        XY[(16 * mt + gq) * kPad + 8 * nt + 2 * tq + 1] = acc[1];
        XY[(16 * mt + gq + 8) * kPad + 8 * nt + 2 * tq] = acc[2];
        XY[(16 * mt + gq + 8) * kPad + 8 * nt + 2 * tq + 1] = acc[3];
    }
    __syncthreads();
    // T[32:64, 0:32] = -T[32:64, 32:64] Y
    {
        const int mt = warp >> 2, nt = warp & 3;
        float acc[4];
        tile_mma(T32, true, 32 + 16 * mt, 32, XY, false, 0, 8 * nt, 4, acc);
        *f32_at(T32, 32 + 16 * mt + gq, 8 * nt + 2 * tq) = -acc[0];
        *f32_at(T32, 32 + 16 * mt + gq, 8 * nt + 2 * tq + 1) = -acc[1];
        *f32_at(T32, 32 + 16 * mt + gq + 8, 8 * nt + 2 * tq) = -acc[2];
        *f32_at(T32, 32 + 16 * mt + gq + 8, 8 * nt + 2 * tq + 1) = -acc[3];
    }
    __syncthreads();
}

}  // namespace chunkc
}  // namespace gdr

namespace gdr {
namespace chunkc {

// Raw inputs of a head for the exact token-by-token fallback.
struct ExactArgs {
    const __nv_bfloat16 *q, *k, *v, *alpha, *b, *w;
    int akind, bkind, wkind;
    __nv_bfloat16* o;
    int T, H, Hq, dv;
};

// Barrier over threads 0..255 only (named barrier 1): the whole block in the
// 256-thread kernels, the compute warps where a further warp issues MMAs.
__device__ __forceinline__ void compute_bar() {
    asm volatile("bar.sync 1, 256;" ::: "memory");
}

// In lane l, the sum over the warp's 32 lanes of x[l] (a reduce-scatter by
// recursive halving: 31 shuffles for 32 columns). x is destroyed.
__device__ __forceinline__ float warp_colsum32(float* x, int lane) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = up ? x[i] : x[i + off];
            const float keep = up ? x[i + off] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return x[0];
}

// Tokens [t0, t0 + n) of head (bb, h) applied exactly in fp32 to the block's
// 128 x (2 NPT) state slice (thread: state row `row` = tid & 127, columns
// v0 + wg * NPT + 0..NPT-1 in S[NPT], wg = tid >> 7), token by token as the
// recurrence defines it: S <- Diag(alpha) S; r = (b.k) S; S <- S - k^T r +
// (w.k)^T v; o = q S. Writes o of those tokens and columns. Used for a chunk
// whose decay span is outside what the tensor-core factorisation can hold.
// Threads 0..255; red is shared scratch of 18 NPT floats; ends with a barrier.
template <int NPT>
__device__ __forceinline__ void exact_tokens(const ExactArgs& a, float (&S)[NPT], float* red, int bb,
                                             int h, int hq, int v0, int t0, int n, int tid) {
    static_assert(NPT % 32 == 0, "columns per thread: a multiple of 32");
    const int row = tid & 127, wg = tid >> 7, w4 = (tid >> 5) & 3, lane = tid & 31;
    float* redR = red;                 // [2][4][NPT] per-warp partial sums
    float* redO = red + 8 * NPT;       // [2][4][NPT]
    float* r2 = red + 16 * NPT;        // [2][NPT] erase reads r
    auto bf = [](__nv_bfloat16 x) { return __bfloat162float(x); };
    for (int tt = 0; tt < n; ++tt) {
        const int t = t0 + tt;
        const size_t tk = ((size_t)bb * a.T + t) * a.H + h;
        const size_t tq = ((size_t)bb * a.T + t) * a.Hq + hq;
        const float kr = bf(a.k[tq * DK + row]), qr = bf(a.q[tq * DK + row]);
        const float ar = a.akind == GDR_GATE_CHANNEL ? bf(a.alpha[tk * DK + row])
                         : a.akind == GDR_GATE_SCALAR ? bf(a.alpha[tk]) : 1.f;
        const float br = a.bkind == GDR_GATE_CHANNEL ? bf(a.b[tk * DK + row])
                         : a.bkind == GDR_GATE_SCALAR ? bf(a.b[tk]) : 0.f;
        const float wr = a.wkind == GDR_GATE_TIED ? br
                         : a.wkind == GDR_GATE_CHANNEL ? bf(a.w[tk * DK + row])
                         : a.wkind == GDR_GATE_SCALAR ? bf(a.w[tk]) : 1.f;
        const uint4* vp = reinterpret_cast<const uint4*>(a.v + tk * a.dv + v0 + wg * NPT);
        // decay, then the erase read r = (b.k) S over the 128 rows
        const float er = br * kr;
#pragma unroll
        for (int g = 0; g < NPT / 32; ++g) {
            float x[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                S[g * 32 + j] *= ar;
                x[j] = er * S[g * 32 + j];
            }
            redR[(wg * 4 + w4) * NPT + g * 32 + lane] = warp_colsum32(x, lane);
        }
        compute_bar();
        if (w4 == 0) {
#pragma unroll
            for (int g = 0; g < NPT / 32; ++g) {
                const int c = g * 32 + lane;
                r2[wg * NPT + c] = redR[(wg * 4) * NPT + c] + redR[(wg * 4 + 1) * NPT + c] +
                                   redR[(wg * 4 + 2) * NPT + c] + redR[(wg * 4 + 3) * NPT + c];
            }
        }
        compute_bar();
        // erase along k, write with key w.k, then the read o = q S
        const float ur = wr * kr;
#pragma unroll
        for (int g = 0; g < NPT / 32; ++g) {
            float v[32], x[32];  // 32 columns of v at a time
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 u = vp[g * 4 + c];
                const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(hh[e]);
                    v[c * 8 + 2 * e] = f.x;
                    v[c * 8 + 2 * e + 1] = f.y;
                }
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int c = g * 32 + j;
                S[c] = fmaf(-kr, r2[wg * NPT + c], fmaf(ur, v[j], S[c]));
                x[j] = qr * S[c];
            }
            redO[(wg * 4 + w4) * NPT + g * 32 + lane] = warp_colsum32(x, lane);
        }
        compute_bar();
        if (w4 == 0) {
#pragma unroll
            for (int g = 0; g < NPT / 32; ++g) {
                const int c = g * 32 + lane;
                const float ov = redO[(wg * 4) * NPT + c] + redO[(wg * 4 + 1) * NPT + c] +
                                 redO[(wg * 4 + 2) * NPT + c] + redO[(wg * 4 + 3) * NPT + c];
                a.o[tk * a.dv + v0 + wg * NPT + c] = __float2bfloat16_rn(ov);
            }
        }
    }
    compute_bar();
}

}  // namespace chunkc
}  // namespace gdr
