// Backward pass of the gated delta rule: fp32 arithmetic on CUDA cores.
//
// The pages ask for a gate-aware backward pass ("Erase-then-Delta Attention"
// (Gated DeltaNet-2), abstract) without printing one. This is reverse-mode
// differentiation of the token recurrence
//   S' = Diag(alpha_t) S_{t-1},  r_t = (b_t . k_t) S',
//   S_t = S' - k_t^T r_t + (w_t . k_t)^T v_t,  o_t = q_t S_t
// ("Recurrent Memory: Write, Erase, Decay, Read", sections 01-05), from the
// last token to the first with G = dL/dS_t (e = b.k, u = w.k):
//   dq_t = dO_t S_t^T,   G += q_t^T dO_t,
//   dv_t = u G,  dr_t = -k G,  du = G v_t^T,  dk = -G r_t^T,
//   de = S' dr_t^T,  dS' = G + e^T dr_t,  dalpha = rowsum(dS' . S_{t-1}),
//   G <- Diag(alpha_t) dS',  dk += b.de + w.du,  db = k.de,  dw = k.du.
//
// Structure. The state gradient obeys its own recurrence,
//   G_{t-1} = Diag(alpha_t) (I - e_t^T k_t) G_t + q_{t-1}^T dO_{t-1},
// which never reads S, so the two sequential parts are independent scans:
//  1. bwd_scan_staged_kernel (bwd_scan_kernel when a d_k row is not a whole
//     number of 16-byte pieces), one warp per 8 state columns of a head (the
//     column sums over d_k are in-thread plus warp shuffles): forward over
//     the tokens: the state at every 64-token chunk start and r_t of every
//     token; backward over the tokens: G at every chunk end, dr_t and dv_t
//     of every token, and dS0. Both directions run in one launch.
//  2. bwd_chunk_kernel, parallel over (row block, chunk, head): from the
//     chunk's start state and end gradient it rebuilds S_{t-1} (elementwise,
//     with r_t known; two levels: states at 8-token sub-chunk starts in
//     shared memory, then 8 states in registers) and G_t (elementwise, with
//     dr_t known), and forms dq, dk and the gate gradients. A CTA holds
//     whole rows of the state, so the sums over columns stay inside it.
//  3. bwd_gate_sum_kernel (scalar gates only): the sum over key channels of a
//     scalar gate's gradient, from the per-row-block partial sums of pass 2;
//     bwd_group_sum_kernel (grouped heads only): dq, dk of each q/k head
//     summed over the value heads that share it.
// The Gated DeltaNet form in bf16 at d_k = d_v = 128 runs every part on
// tensor cores instead: the forward two-pass kernels checkpoint the state at
// every chunk start and U = beta v - r of every token, the chunkwise
// state-gradient pass (chunk_bwd_grad_sm100.cu) gives G at every chunk end,
// dr, dv and dS0, and the tensor-core chunk kernel (chunk_bwd_tc_sm100.cu)
// the other gradients.
#include "common.cuh"

namespace gdr {
cudaError_t launch_bwd_chunk_tc(const CUtensorMap* maps, const CUtensorMap* ck_maps, const void* alpha,
                                const void* beta, float* dq, float* dk, float* dalpha, float* db,
                                int* d_status, int B, int T, int H, int group, int nchunks,
                                cudaStream_t st);
bool make_tma_map_bf16(CUtensorMap* m, const void* base, int B, int T, int H, int d);
bool make_tma_map_f32(CUtensorMap* m, const void* base, int B, int T, int H, int d);
size_t twopass_workspace_bytes(int B, int T, int H, int dv);
cudaError_t launch_chunk_twopass_gdn(const CUtensorMap* maps, const CUtensorMap* ws_maps, void* ws,
                                     const void* alpha, const void* beta, const float* S0, void* o,
                                     float* ST, int* d_status, int B, int T, int H, int dv, int group,
                                     cudaStream_t st, __nv_bfloat16* ckS, __nv_bfloat16* up);
cudaError_t launch_bwd_grad_tc(const CUtensorMap* q_map, const CUtensorMap* k_map, const CUtensorMap* do_map,
                               const CUtensorMap* ws_maps, const void* alpha, const void* beta,
                               const float* dST, __nv_bfloat16* ckG, __nv_bfloat16* DR, float* dv, float* dS0,
                               int* d_status, int B, int T, int H, int dvn, int group, cudaStream_t st);

namespace bwd {

constexpr int kC = 64;           // chunk: checkpoint interval of the scans
constexpr int kSub = 8;          // sub-chunk: states rebuilt in registers
constexpr int kNSub = kC / kSub;
constexpr int kMaxDK = 256;      // 4 rows per lane in the scans up to d_k = 128, 8 beyond
constexpr int kStagedMaxDK = 128; // the staged scan's shared-memory rows
constexpr int kMaxDV = 256;      // 8 columns per thread, up to 32 threads per row in pass 2
constexpr int kScanWarps = 4;    // scan CTA: 4 warps
constexpr int kScanCols = 8;     // state columns per scan warp
constexpr int kChunkThreads = 128;

struct Params {
    const void *q, *k, *v, *alpha, *b, *w, *dO;
    const float *S0, *dST;
    float *dq, *dk, *dv, *dalpha, *db, *dw, *dS0;
    float *ckS, *ckG, *R, *DR, *GP;  // workspace
    int* d_status;                   // bounded waits of the tensor-core kernels
    float *dq_out, *dk_out;          // grouped heads: the caller's dq, dk (dq, dk are then workspace)
    int B, T, H, Hq, group, dk_, dv_, akind, bkind, wkind, nchunks, tpr, nrb;
};

template <typename TI>
__device__ __forceinline__ float ld1(const void* p, size_t i) {
    return to_f32(static_cast<const TI*>(p)[i]);
}

template <typename TI>
__device__ __forceinline__ void load4(const void* p, size_t off, float (&x)[4]);
template <>
__device__ __forceinline__ void load4<float>(const void* p, size_t off, float (&x)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(p) + off);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const void* p, size_t off, float (&x)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(p) + off);
    x[0] = __uint_as_float(u.x << 16); x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16); x[3] = __uint_as_float(u.y & 0xffff0000u);
}

template <typename TI>
__device__ __forceinline__ void load8(const void* p, size_t off, float (&x)[8]) {
    float a[4], b[4];
    load4<TI>(p, off, a);
    load4<TI>(p, off + 4, b);
#pragma unroll
    for (int c = 0; c < 4; ++c) { x[c] = a[c]; x[4 + c] = b[c]; }
}

__device__ __forceinline__ void store4(float* dst, const float (&x)[4]) {
    *reinterpret_cast<float4*>(dst) = make_float4(x[0], x[1], x[2], x[3]);
}

// Per-row scalars of one token for key channel i (neutral beyond d_k).
struct Row {
    float q, k, a, bg, wg;
};

// tok indexes the value head's [B, T, H] token, tokq the q/k head's [B, T, H_qk] one.
template <typename TI>
__device__ __forceinline__ Row load_row(const Params& p, size_t tok, size_t tokq, int i) {
    Row r{0.f, 0.f, 1.f, 0.f, 0.f};
    if (i < p.dk_) {
        const size_t gi = tok * p.dk_ + i;
        r.q = ld1<TI>(p.q, tokq * p.dk_ + i);
        r.k = ld1<TI>(p.k, tokq * p.dk_ + i);
        if (p.akind == GDR_GATE_SCALAR) r.a = ld1<TI>(p.alpha, tok);
        else if (p.akind == GDR_GATE_CHANNEL) r.a = ld1<TI>(p.alpha, gi);
        if (p.bkind == GDR_GATE_SCALAR) r.bg = ld1<TI>(p.b, tok);
        else if (p.bkind == GDR_GATE_CHANNEL) r.bg = ld1<TI>(p.b, gi);
        if (p.wkind == GDR_GATE_TIED) r.wg = r.bg;
        else if (p.wkind == GDR_GATE_NONE) r.wg = 1.f;
        else if (p.wkind == GDR_GATE_SCALAR) r.wg = ld1<TI>(p.w, tok);
        else r.wg = ld1<TI>(p.w, gi);
    }
    return r;
}

// Warp sum of NV values per lane, all lanes receiving all NV totals:
// halving exchanges (each lane keeps the half its partner does not), plain
// sums over the remaining lanes, then a broadcast of each total.
template <int NV>
__device__ __forceinline__ void warp_allsum(float (&x)[NV], int lane) {
    float y[NV];
#pragma unroll
    for (int v = 0; v < NV; ++v) y[v] = x[v];
    int off = 16;
#pragma unroll
    for (int half = NV / 2; half >= 1; half >>= 1, off >>= 1) {
        const bool hi = (lane & off) != 0;
#pragma unroll
        for (int v = 0; v < half; ++v) {
            const float send = hi ? y[v] : y[v + half];
            const float keep = hi ? y[v + half] : y[v];
            y[v] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    float s = y[0];
#pragma unroll
    for (; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    // lane l now holds the total of value (l / (32 / NV))
#pragma unroll
    for (int v = 0; v < NV; ++v) x[v] = __shfl_sync(0xffffffffu, s, v * (32 / NV));
}

// Per-row scalars of rows i0 .. i0 + R - 1 of one token (neutral beyond d_k).
// With d_k a multiple of 4 every four rows are one vector load per input.
template <int R>
struct RowsR {
    float q[R], k[R], a[R], bg[R], wg[R];
};
using Rows4 = RowsR<4>;

template <typename TI, int R>
__device__ __forceinline__ void load_rows(const Params& p, size_t tok, size_t tokq, int i0, RowsR<R>& r) {
    if ((p.dk_ & 3) == 0) {
#pragma unroll
        for (int g = 0; g < R; g += 4) {
            const int ig = i0 + g;
            if (ig < p.dk_) {
                const size_t gi = tok * p.dk_ + ig;
                load4<TI>(p.q, tokq * p.dk_ + ig, *reinterpret_cast<float(*)[4]>(r.q + g));
                load4<TI>(p.k, tokq * p.dk_ + ig, *reinterpret_cast<float(*)[4]>(r.k + g));
                if (p.akind == GDR_GATE_CHANNEL) load4<TI>(p.alpha, gi, *reinterpret_cast<float(*)[4]>(r.a + g));
                else {
                    const float a = p.akind == GDR_GATE_SCALAR ? ld1<TI>(p.alpha, tok) : 1.f;
                    r.a[g] = r.a[g + 1] = r.a[g + 2] = r.a[g + 3] = a;
                }
                if (p.bkind == GDR_GATE_CHANNEL) load4<TI>(p.b, gi, *reinterpret_cast<float(*)[4]>(r.bg + g));
                else {
                    const float bb = p.bkind == GDR_GATE_SCALAR ? ld1<TI>(p.b, tok) : 0.f;
                    r.bg[g] = r.bg[g + 1] = r.bg[g + 2] = r.bg[g + 3] = bb;
                }
                if (p.wkind == GDR_GATE_CHANNEL) load4<TI>(p.w, gi, *reinterpret_cast<float(*)[4]>(r.wg + g));
                else if (p.wkind == GDR_GATE_TIED) {
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) r.wg[g + rr] = r.bg[g + rr];
                } else {
                    const float ww = p.wkind == GDR_GATE_SCALAR ? ld1<TI>(p.w, tok) : 1.f;
                    r.wg[g] = r.wg[g + 1] = r.wg[g + 2] = r.wg[g + 3] = ww;
                }
            } else {
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    r.q[g + rr] = r.k[g + rr] = r.bg[g + rr] = r.wg[g + rr] = 0.f;
                    r.a[g + rr] = 1.f;
                }
            }
        }
        return;
    }
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
        const Row w1 = load_row<TI>(p, tok, tokq, i0 + rr);
        r.q[rr] = w1.q; r.k[rr] = w1.k; r.a[rr] = w1.a; r.bg[rr] = w1.bg; r.wg[rr] = w1.wg;
    }
}

template <typename TI>
__device__ __forceinline__ void load_rows4(const Params& p, size_t tok, size_t tokq, int i0, Rows4& r) {
    load_rows<TI, 4>(p, tok, tokq, i0, r);
}

// ----------------------------------------------------------------- pass 1 --
// blockIdx.z = 2 b + direction; warp w of CTA x owns columns
// 8 (kScanWarps x + w) .. + 8 (those below d_v), lane l owns rows R l .. R l + R - 1
// (R = 4 up to d_k = 128, 8 up to d_k = 256).
template <typename TI, int R>
__global__ void __launch_bounds__(kScanWarps * 32) bwd_scan_kernel(Params p) {
    constexpr int NC = kScanCols;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c0 = NC * (kScanWarps * blockIdx.x + warp);
    if (c0 >= p.dv_) return;  // no block-wide barriers in this kernel
    const int b = (int)(blockIdx.z >> 1);
    const int dir = (int)(blockIdx.z & 1), h = blockIdx.y;
    const size_t head = (size_t)b * p.H + h;
    const int i0 = R * lane;
    auto tok_of = [&](int t) { return ((size_t)b * p.T + t) * p.H + h; };
    const int hq = h / p.group;
    auto tokq_of = [&](int t) { return ((size_t)b * p.T + t) * p.Hq + hq; };
    auto ck_at = [&](float* base, int chunk, int i) {
        return base + ((head * p.nchunks + chunk) * p.dk_ + i) * p.dv_ + c0;
    };
    float X[R][NC];  // S (forward) or G (backward): rows i0 + rr, columns c0 + c
    const float* init = dir == 0 ? p.S0 : p.dST;
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
        if (init && i0 + rr < p.dk_) load8<float>(init, (head * p.dk_ + i0 + rr) * p.dv_ + c0, X[rr]);
        else
            for (int c = 0; c < NC; ++c) X[rr][c] = 0.f;
    }
    // the next token's inputs are loaded while the current one is computed
    const void* colsrc = dir == 0 ? p.v : p.dO;
    RowsR<R> nrw;
    float nvec[NC];
    const int tfirst = dir == 0 ? 0 : p.T - 1;
    load_rows<TI, R>(p, tok_of(tfirst), tokq_of(tfirst), i0, nrw);
    load8<TI>(colsrc, tok_of(tfirst) * p.dv_ + c0, nvec);
    for (int n = 0; n < p.T; ++n) {
        const int t = dir == 0 ? n : p.T - 1 - n;
        const size_t tok = tok_of(t);
        const bool store_ck = dir == 0 ? (t % kC == 0) : (t == p.T - 1 || (t + 1) % kC == 0);
        if (store_ck)  // forward: chunk start; backward: before the chunk's last token
#pragma unroll
            for (int rr = 0; rr < R; ++rr)
                if (i0 + rr < p.dk_) {
                    float* dst = ck_at(dir == 0 ? p.ckS : p.ckG, t / kC, i0 + rr);
                    reinterpret_cast<float4*>(dst)[0] = make_float4(X[rr][0], X[rr][1], X[rr][2], X[rr][3]);
                    reinterpret_cast<float4*>(dst)[1] = make_float4(X[rr][4], X[rr][5], X[rr][6], X[rr][7]);
                }
        const RowsR<R> rw = nrw;
        float cv[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) cv[c] = nvec[c];
        if (n + 1 < p.T) {
            const int tnext = dir == 0 ? t + 1 : t - 1;
            const size_t tn = tok_of(tnext);
            load_rows<TI, R>(p, tn, tokq_of(tnext), i0, nrw);
            load8<TI>(colsrc, tn * p.dv_ + c0, nvec);
        }
        if (dir == 0) {
            // S' = Diag(a) S; r = e S' (sum over rows); S = S' - k^T r + u^T v
            float r[NC];
#pragma unroll
            for (int c = 0; c < NC; ++c) r[c] = 0.f;
#pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                const float e = rw.bg[rr] * rw.k[rr];
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    X[rr][c] *= rw.a[rr];
                    r[c] = fmaf(e, X[rr][c], r[c]);
                }
            }
            warp_allsum<NC>(r, lane);
#pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                const float u = rw.wg[rr] * rw.k[rr];
#pragma unroll
                for (int c = 0; c < NC; ++c)
                    X[rr][c] = fmaf(-rw.k[rr], r[c], fmaf(u, cv[c], X[rr][c]));
            }
            if (lane == 0) {
                float* dst = p.R + tok * p.dv_ + c0;
                reinterpret_cast<float4*>(dst)[0] = make_float4(r[0], r[1], r[2], r[3]);
                reinterpret_cast<float4*>(dst)[1] = make_float4(r[4], r[5], r[6], r[7]);
            }
        } else {
            // G += q^T dO; dr = -k G, dv = u G (sums over rows); G = Diag(a) (G + e^T dr)
            float z[2 * NC];  // k G | u G
#pragma unroll
            for (int c = 0; c < 2 * NC; ++c) z[c] = 0.f;
#pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                const float u = rw.wg[rr] * rw.k[rr];
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    X[rr][c] = fmaf(rw.q[rr], cv[c], X[rr][c]);
                    z[c] = fmaf(rw.k[rr], X[rr][c], z[c]);
                    z[NC + c] = fmaf(u, X[rr][c], z[NC + c]);
                }
            }
            warp_allsum<2 * NC>(z, lane);
#pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                const float e = rw.bg[rr] * rw.k[rr];
#pragma unroll
                for (int c = 0; c < NC; ++c) X[rr][c] = rw.a[rr] * fmaf(-e, z[c], X[rr][c]);
            }
            if (lane == 0) {
                float* dst = p.DR + tok * p.dv_ + c0;
                reinterpret_cast<float4*>(dst)[0] = make_float4(-z[0], -z[1], -z[2], -z[3]);
                reinterpret_cast<float4*>(dst)[1] = make_float4(-z[4], -z[5], -z[6], -z[7]);
                float* dvp = p.dv + tok * p.dv_ + c0;
                reinterpret_cast<float4*>(dvp)[0] = make_float4(z[8], z[9], z[10], z[11]);
                reinterpret_cast<float4*>(dvp)[1] = make_float4(z[12], z[13], z[14], z[15]);
            }
        }
    }
    if (dir == 1 && p.dS0)
#pragma unroll
        for (int rr = 0; rr < R; ++rr)
            if (i0 + rr < p.dk_) {
                float* dst = p.dS0 + (head * p.dk_ + i0 + rr) * p.dv_ + c0;
                reinterpret_cast<float4*>(dst)[0] = make_float4(X[rr][0], X[rr][1], X[rr][2], X[rr][3]);
                reinterpret_cast<float4*>(dst)[1] = make_float4(X[rr][4], X[rr][5], X[rr][6], X[rr][7]);
            }
}

// Staged form of pass 1, used when a token's d_k-row of q / k / channel gate
// is a whole number of 16-byte pieces: the CTA's four warps (one head, 32
// columns) share the row scalars, so the CTA copies blocks of kNT tokens
// into shared memory with cp.async, one block ahead of the one it computes
// (double buffer), instead of every lane loading its rows per token.
constexpr int kNT = 8;

template <typename TI>
struct ScanStage {
    TI rows[5][kNT][kStagedMaxDK];            // q, k, alpha, b, w (channel kinds)
    TI cols[kNT][kScanWarps * kScanCols];     // v (forward) or dO (backward)
    float scal[3][kNT];                       // scalar alpha, b, w
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_prev() {  // all but the most recent group landed
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}

template <typename TI>
__device__ __forceinline__ void lds4(const TI* src, float (&x)[4]);
template <>
__device__ __forceinline__ void lds4<float>(const float* src, float (&x)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(src);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}
template <>
__device__ __forceinline__ void lds4<__nv_bfloat16>(const __nv_bfloat16* src, float (&x)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    x[0] = __uint_as_float(u.x << 16); x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16); x[3] = __uint_as_float(u.y & 0xffff0000u);
}

template <typename TI>
__global__ void __launch_bounds__(kScanWarps * 32) bwd_scan_staged_kernel(Params p) {
    constexpr int NC = kScanCols;
    constexpr int CTA_COLS = kScanWarps * NC;
    auto st_cols = [](float* dst, const float* x, float sign) {  // NC columns, 16-byte stores
#pragma unroll
        for (int c = 0; c < NC; c += 4)
            *reinterpret_cast<float4*>(dst + c) =
                make_float4(sign * x[c], sign * x[c + 1], sign * x[c + 2], sign * x[c + 3]);
    };
    __shared__ __align__(16) ScanStage<TI> stg[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cb = CTA_COLS * blockIdx.x;  // the CTA's first column
    const int c0 = cb + NC * warp;
    const bool active = c0 < p.dv_;       // idle warps still copy and meet the barriers
    const int ncols = min(CTA_COLS, p.dv_ - cb);
    const int b = (int)(blockIdx.z >> 1);
    const int dir = (int)(blockIdx.z & 1), h = blockIdx.y;
    const size_t head = (size_t)b * p.H + h;
    const int i0 = 4 * lane;
    const bool rows_ok = i0 < p.dk_;       // d_k is a multiple of 4 here
    auto tok_of = [&](int t) { return ((size_t)b * p.T + t) * p.H + h; };
    auto tok_n = [&](int n) { return tok_of(dir == 0 ? n : p.T - 1 - n); };
    const int hq = h / p.group;
    auto tokq_n = [&](int n) { return ((size_t)b * p.T + (dir == 0 ? n : p.T - 1 - n)) * p.Hq + hq; };
    const void* colsrc = dir == 0 ? p.v : p.dO;
    // vectors copied per token: q (backward only), k, and the channel gates
    const void* vsrc[5] = {p.q, p.k, p.alpha, p.b, p.w};
    bool vneed[5] = {dir == 1, true, p.akind == GDR_GATE_CHANNEL, p.bkind == GDR_GATE_CHANNEL,
                     p.wkind == GDR_GATE_CHANNEL};
    constexpr int EPC = 16 / sizeof(TI);  // elements per 16-byte piece
    const int row_pieces = p.dk_ / EPC, col_pieces = ncols / EPC;

    auto issue = [&](int blk, int buf) {
        const int n0 = blk * kNT, nt = min(kNT, p.T - n0);
        for (int vi = 0; vi < 5; ++vi) {
            if (!vneed[vi]) continue;
            for (int idx = tid; idx < nt * row_pieces; idx += kScanWarps * 32) {
                const int tt = idx / row_pieces, pc = idx % row_pieces;
                const size_t tk = vi < 2 ? tokq_n(n0 + tt) : tok_n(n0 + tt);  // q, k: q/k head
                cp_async16(&stg[buf].rows[vi][tt][pc * EPC],
                           static_cast<const TI*>(vsrc[vi]) + tk * p.dk_ + pc * EPC);
            }
        }
        for (int idx = tid; idx < nt * col_pieces; idx += kScanWarps * 32) {
            const int tt = idx / col_pieces, pc = idx % col_pieces;
            cp_async16(&stg[buf].cols[tt][pc * EPC],
                       static_cast<const TI*>(colsrc) + tok_n(n0 + tt) * p.dv_ + cb + pc * EPC);
        }
        cp_async_commit();
    };
    // scalar gates: thread tt < kNT loads token tt of a block into registers
    auto load_scal = [&](int blk, float (&sc)[3]) {
        const int n = blk * kNT + tid;
        sc[0] = 1.f; sc[1] = 0.f; sc[2] = 1.f;
        if (tid < kNT && n < p.T) {
            const size_t tok = tok_n(n);
            if (p.akind == GDR_GATE_SCALAR) sc[0] = ld1<TI>(p.alpha, tok);
            if (p.bkind == GDR_GATE_SCALAR) sc[1] = ld1<TI>(p.b, tok);
            if (p.wkind == GDR_GATE_SCALAR) sc[2] = ld1<TI>(p.w, tok);
        }
    };
    auto store_scal = [&](int buf, const float (&sc)[3]) {
        if (tid < kNT)
#pragma unroll
            for (int g = 0; g < 3; ++g) stg[buf].scal[g][tid] = sc[g];
    };

    float X[4][NC];
    const float* init = dir == 0 ? p.S0 : p.dST;
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        if (active && init && i0 + rr < p.dk_) {
#pragma unroll
            for (int c = 0; c < NC; c += 4) {
                float x4[4];
                load4<float>(init, (head * p.dk_ + i0 + rr) * p.dv_ + c0 + c, x4);
                X[rr][c] = x4[0]; X[rr][c + 1] = x4[1]; X[rr][c + 2] = x4[2]; X[rr][c + 3] = x4[3];
            }
        } else
            for (int c = 0; c < NC; ++c) X[rr][c] = 0.f;
    }

    const int nblk = (p.T + kNT - 1) / kNT;
    {
        float sc[3];
        load_scal(0, sc);
        store_scal(0, sc);
    }
    issue(0, 0);
    for (int blk = 0; blk < nblk; ++blk) {
        const int buf = blk & 1;
        float scn[3];
        if (blk + 1 < nblk) {
            issue(blk + 1, buf ^ 1);
            load_scal(blk + 1, scn);
        } else {
            cp_async_commit();  // empty group keeps the wait count uniform
        }
        cp_async_wait_prev();
        __syncthreads();  // block blk visible to every thread
        const ScanStage<TI>& S_ = stg[buf];
        const int n0 = blk * kNT, nt = min(kNT, p.T - n0);
        if (active) {
            for (int tt = 0; tt < nt; ++tt) {
                const int t = dir == 0 ? n0 + tt : p.T - 1 - (n0 + tt);
                const size_t tok = tok_of(t);
                const bool store_ck = dir == 0 ? (t % kC == 0) : (t == p.T - 1 || (t + 1) % kC == 0);
                if (store_ck)
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr)
                        if (i0 + rr < p.dk_) {
                            float* dst = (dir == 0 ? p.ckS : p.ckG) +
                                  ((head * p.nchunks + t / kC) * p.dk_ + i0 + rr) * p.dv_ + c0;
                            st_cols(dst, X[rr], 1.f);
                        }
                Rows4 rw;
                if (rows_ok) {
                    if (dir == 1) lds4<TI>(&S_.rows[0][tt][i0], rw.q);
                    lds4<TI>(&S_.rows[1][tt][i0], rw.k);
                    if (vneed[2]) lds4<TI>(&S_.rows[2][tt][i0], rw.a);
                    else rw.a[0] = rw.a[1] = rw.a[2] = rw.a[3] = S_.scal[0][tt];
                    if (vneed[3]) lds4<TI>(&S_.rows[3][tt][i0], rw.bg);
                    else rw.bg[0] = rw.bg[1] = rw.bg[2] = rw.bg[3] = S_.scal[1][tt];
                    if (p.wkind == GDR_GATE_TIED) {
#pragma unroll
                        for (int rr = 0; rr < 4; ++rr) rw.wg[rr] = rw.bg[rr];
                    } else if (vneed[4]) lds4<TI>(&S_.rows[4][tt][i0], rw.wg);
                    else rw.wg[0] = rw.wg[1] = rw.wg[2] = rw.wg[3] = S_.scal[2][tt];
                    if (dir == 0) rw.q[0] = rw.q[1] = rw.q[2] = rw.q[3] = 0.f;
                } else {
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        rw.q[rr] = rw.k[rr] = rw.bg[rr] = rw.wg[rr] = 0.f;
                        rw.a[rr] = 1.f;
                    }
                }
                float cv[NC];
#pragma unroll
                for (int c = 0; c < NC; c += 4) {
                    float a4[4];
                    lds4<TI>(&S_.cols[tt][NC * warp + c], a4);
                    cv[c] = a4[0]; cv[c + 1] = a4[1]; cv[c + 2] = a4[2]; cv[c + 3] = a4[3];
                }
                if (dir == 0) {
                    float r[NC];
#pragma unroll
                    for (int c = 0; c < NC; ++c) r[c] = 0.f;
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        const float e = rw.bg[rr] * rw.k[rr];
#pragma unroll
                        for (int c = 0; c < NC; ++c) {
                            X[rr][c] *= rw.a[rr];
                            r[c] = fmaf(e, X[rr][c], r[c]);
                        }
                    }
                    warp_allsum<NC>(r, lane);
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        const float u = rw.wg[rr] * rw.k[rr];
#pragma unroll
                        for (int c = 0; c < NC; ++c)
                            X[rr][c] = fmaf(-rw.k[rr], r[c], fmaf(u, cv[c], X[rr][c]));
                    }
                    if (lane == 0) {
                        st_cols(p.R + tok * p.dv_ + c0, r, 1.f);
                    }
                } else {
                    float z[2 * NC];
#pragma unroll
                    for (int c = 0; c < 2 * NC; ++c) z[c] = 0.f;
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        const float u = rw.wg[rr] * rw.k[rr];
#pragma unroll
                        for (int c = 0; c < NC; ++c) {
                            X[rr][c] = fmaf(rw.q[rr], cv[c], X[rr][c]);
                            z[c] = fmaf(rw.k[rr], X[rr][c], z[c]);
                            z[NC + c] = fmaf(u, X[rr][c], z[NC + c]);
                        }
                    }
                    warp_allsum<2 * NC>(z, lane);
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        const float e = rw.bg[rr] * rw.k[rr];
#pragma unroll
                        for (int c = 0; c < NC; ++c) X[rr][c] = rw.a[rr] * fmaf(-e, z[c], X[rr][c]);
                    }
                    if (lane == 0) {
                        st_cols(p.DR + tok * p.dv_ + c0, z, -1.f);
                        st_cols(p.dv + tok * p.dv_ + c0, z + NC, 1.f);
                    }
                }
            }
        }
        if (blk + 1 < nblk) store_scal(buf ^ 1, scn);
        __syncthreads();  // buffer blk is reused by the copies issued next
    }
    if (active && dir == 1 && p.dS0)
#pragma unroll
        for (int rr = 0; rr < 4; ++rr)
            if (i0 + rr < p.dk_) {
                st_cols(p.dS0 + (head * p.dk_ + i0 + rr) * p.dv_ + c0, X[rr], 1.f);
            }
}

// ----------------------------------------------------------------- pass 2 --
// CTA (row block, chunk, head). Thread t: row rb * RB + t / tpr, columns
// 8 (t % tpr) .. + 8, with tpr threads per row (a power of two <= 32, so a
// row's threads share a warp) and RB = 128 / tpr rows per CTA. A sub-chunk's
// inputs (row scalars of the CTA's rows, v, dO, r, dr over all columns) are
// staged in shared memory as fp32 by the whole CTA before it is used.
struct ChunkSmem {
    // byte offsets into the dynamic shared memory
    uint32_t subck, col, row, sred, total;
    int dvp, RB;
};

__host__ __device__ inline ChunkSmem chunk_smem(int tpr) {
    ChunkSmem m;
    m.dvp = 8 * tpr;
    m.RB = kChunkThreads / tpr;
    m.subck = 0;                                                    // [kNSub][2][128] float4
    m.col = m.subck + kNSub * 2 * kChunkThreads * 16;               // [4][kSub][dvp] fp32
    m.row = m.col + 4 * kSub * m.dvp * 4;                           // [kSub][5][RB] fp32
    m.sred = m.row + kSub * 5 * m.RB * 4;                           // [kSub][3][4] fp32
    m.total = m.sred + kSub * 3 * (kChunkThreads / 32) * 4;
    return m;
}

enum { kV = 0, kDO = 1, kR = 2, kDR = 3 };

template <typename TI>
__global__ void __launch_bounds__(kChunkThreads, 4) bwd_chunk_kernel(Params p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int tpr = p.tpr;
    const ChunkSmem L = chunk_smem(tpr);
    float4* subck = reinterpret_cast<float4*>(smem_raw + L.subck);
    float* colb = reinterpret_cast<float*>(smem_raw + L.col);
    float* rowb = reinterpret_cast<float*>(smem_raw + L.row);
    float* sred = reinterpret_cast<float*>(smem_raw + L.sred);
    const int dvp = L.dvp, RB = L.RB;
    auto col_at = [&](int a, int u) { return colb + (a * kSub + u) * dvp; };
    auto row_at = [&](int u, int qy) { return rowb + (u * 5 + qy) * RB; };

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = tid & (tpr - 1), lr = tid / tpr;
    const int rb = blockIdx.x, c = blockIdx.y;
    const int bh = blockIdx.z, b = bh / p.H, h = bh % p.H;
    const size_t head = (size_t)bh;
    const int i = rb * RB + lr;
    // columns 4 g .. 4 g + 3 and 4 (g + tpr) .. + 3: a row's threads read
    // consecutive 16-byte pieces of a staged row (no bank conflicts)
    const int ja = 4 * g, jb = 4 * (g + tpr);
    const bool row_ok = i < p.dk_;
    const int t0 = c * kC, Lc = min(kC, p.T - t0);
    auto tok_of = [&](int t) { return ((size_t)b * p.T + t) * p.H + h; };

    // Stage tokens tau0 .. tau0 + ns - 1 of the chunk: the listed column
    // arrays (zero beyond d_v) and the row scalars.
    auto stage = [&](int tau0, int ns, bool bwd) {
        __syncthreads();  // previous contents fully read
        const int n4 = dvp / 4;  // float4 per token row (a power of two, as is RB)
        const int lg_n4 = __ffs(n4) - 1, lg_rb = __ffs(RB) - 1;
        const size_t tok0 = tok_of(t0 + tau0);  // token u of the sub-chunk: tok0 + u H
        const size_t tokq0 = ((size_t)b * p.T + t0 + tau0) * p.Hq + h / p.group;
        const int narr = bwd ? 4 : 2;
        for (int ai = 0; ai < narr; ++ai) {
            const int a = bwd ? ai : (ai == 0 ? kV : kR);
            for (int idx = tid; idx < (kSub << lg_n4); idx += kChunkThreads) {
                const int u = idx >> lg_n4, c4 = (idx & (n4 - 1)) << 2;
                float x[4] = {0.f, 0.f, 0.f, 0.f};
                if (u < ns && c4 < p.dv_) {
                    const size_t off = (tok0 + (size_t)u * p.H) * p.dv_ + c4;
                    if (a == kV) load4<TI>(p.v, off, x);
                    else if (a == kDO) load4<TI>(p.dO, off, x);
                    else load4<float>(a == kR ? p.R : p.DR, off, x);
                }
                *reinterpret_cast<float4*>(col_at(a, u) + c4) = make_float4(x[0], x[1], x[2], x[3]);
            }
        }
        for (int idx = tid; idx < (kSub << lg_rb); idx += kChunkThreads) {
            const int u = idx >> lg_rb, r = idx & (RB - 1);
            Row rw{0.f, 0.f, 1.f, 0.f, 0.f};
            if (u < ns) rw = load_row<TI>(p, tok0 + (size_t)u * p.H, tokq0 + (size_t)u * p.Hq, rb * RB + r);
            row_at(u, 0)[r] = rw.q;
            row_at(u, 1)[r] = rw.k;
            row_at(u, 2)[r] = rw.a;
            row_at(u, 3)[r] = rw.bg;
            row_at(u, 4)[r] = rw.wg;
        }
        __syncthreads();
    };
    auto ld8s = [&](const float* src, float (&x)[8]) {  // this thread's 8 columns of a staged row
        const float4 a = *reinterpret_cast<const float4*>(src + ja);
        const float4 bq = *reinterpret_cast<const float4*>(src + jb);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = bq.x; x[5] = bq.y; x[6] = bq.z; x[7] = bq.w;
    };

    float S[8], G[8];
    {
        // columns at or beyond d_v (and rows beyond d_k) hold zeros and stay zero:
        // their staged inputs are zero and their row scalars neutral
        const size_t off = ((head * p.nchunks + c) * p.dk_ + i) * p.dv_;
        float a4[4], b4[4];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) a4[cc] = b4[cc] = 0.f;
        if (row_ok && ja < p.dv_) load4<float>(p.ckS, off + ja, a4);
        if (row_ok && jb < p.dv_) load4<float>(p.ckS, off + jb, b4);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) { S[cc] = a4[cc]; S[4 + cc] = b4[cc]; }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) a4[cc] = b4[cc] = 0.f;
        if (row_ok && ja < p.dv_) load4<float>(p.ckG, off + ja, a4);
        if (row_ok && jb < p.dv_) load4<float>(p.ckG, off + jb, b4);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) { G[cc] = a4[cc]; G[4 + cc] = b4[cc]; }
    }

    // forward over the chunk: the state at every sub-chunk start
    const int nsub = (Lc + kSub - 1) / kSub;
    for (int s = 0; s < nsub; ++s) {
        const int tau0 = s * kSub, ns = min(kSub, Lc - tau0);
        subck[(s * 2 + 0) * kChunkThreads + tid] = make_float4(S[0], S[1], S[2], S[3]);
        subck[(s * 2 + 1) * kChunkThreads + tid] = make_float4(S[4], S[5], S[6], S[7]);
        if (s == nsub - 1) break;  // the last sub-chunk's start is all the reverse pass needs
        stage(tau0, ns, false);
#pragma unroll
        for (int u = 0; u < kSub; ++u) {
            float v[8], r[8];
            ld8s(col_at(kV, u), v);
            ld8s(col_at(kR, u), r);
            const float a = row_at(u, 2)[lr], kk = row_at(u, 1)[lr], uu = row_at(u, 4)[lr] * kk;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) S[cc] = fmaf(-kk, r[cc], fmaf(uu, v[cc], a * S[cc]));
        }
    }

    for (int s = nsub - 1; s >= 0; --s) {
        const int tau0 = s * kSub, ns = min(kSub, Lc - tau0);
        stage(tau0, ns, true);
        float Sst[kSub + 1][8];  // S_{t-1} of each token, then the state after the last one
        {
            const float4 a0 = subck[(s * 2 + 0) * kChunkThreads + tid];
            const float4 a1 = subck[(s * 2 + 1) * kChunkThreads + tid];
            Sst[0][0] = a0.x; Sst[0][1] = a0.y; Sst[0][2] = a0.z; Sst[0][3] = a0.w;
            Sst[0][4] = a1.x; Sst[0][5] = a1.y; Sst[0][6] = a1.z; Sst[0][7] = a1.w;
        }
#pragma unroll
        for (int u = 0; u < kSub; ++u) {
            float v[8], r[8];
            ld8s(col_at(kV, u), v);
            ld8s(col_at(kR, u), r);
            const float a = row_at(u, 2)[lr], kk = row_at(u, 1)[lr], uu = row_at(u, 4)[lr] * kk;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
                Sst[u + 1][cc] = fmaf(-kk, r[cc], fmaf(uu, v[cc], a * Sst[u][cc]));
        }
#pragma unroll
        for (int u = kSub - 1; u >= 0; --u) {
            if (u < ns) {
                float v[8], d[8], r[8], dr[8];
                ld8s(col_at(kV, u), v);
                ld8s(col_at(kDO, u), d);
                ld8s(col_at(kR, u), r);
                ld8s(col_at(kDR, u), dr);
                const float q = row_at(u, 0)[lr], kk = row_at(u, 1)[lr], a = row_at(u, 2)[lr];
                const float bg = row_at(u, 3)[lr], wg = row_at(u, 4)[lr];
                const float e = bg * kk;
                // partial sums over this thread's 8 columns:
                // dq (S_t dO^T), dk from r (-G r^T), du (G v^T), de (S' dr^T), dalpha
                float acc[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    acc[0] = fmaf(Sst[u + 1][cc], d[cc], acc[0]);
                    G[cc] = fmaf(q, d[cc], G[cc]);
                    acc[1] = fmaf(-G[cc], r[cc], acc[1]);
                    acc[2] = fmaf(G[cc], v[cc], acc[2]);
                    acc[3] = fmaf(a * Sst[u][cc], dr[cc], acc[3]);
                    const float dsd = fmaf(e, dr[cc], G[cc]);
                    acc[4] = fmaf(dsd, Sst[u][cc], acc[4]);
                    G[cc] = a * dsd;
                }
                if (tpr == 16) {
                    // reduce-scatter over the row's 16 lanes (8 slots, 5 used):
                    // lane g ends with the total of slot (g >> 1), then each
                    // total is fetched from its owner
                    float y[8] = {acc[0], acc[1], acc[2], acc[3], acc[4], 0.f, 0.f, 0.f};
#pragma unroll
                    for (int o = 8, half = 4; half >= 1; o >>= 1, half >>= 1) {
                        const bool hi = (g & o) != 0;
#pragma unroll
                        for (int v = 0; v < half; ++v) {
                            const float send = hi ? y[v] : y[v + half];
                            const float keep = hi ? y[v + half] : y[v];
                            y[v] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                        }
                    }
                    const float tot = y[0] + __shfl_xor_sync(0xffffffffu, y[0], 1);
                    const int base = lane & ~15;
#pragma unroll
                    for (int qy = 0; qy < 5; ++qy) acc[qy] = __shfl_sync(0xffffffffu, tot, base + 2 * qy);
                } else {
                    for (int o = 1; o < tpr; o <<= 1)
#pragma unroll
                        for (int qy = 0; qy < 5; ++qy) acc[qy] += __shfl_xor_sync(0xffffffffu, acc[qy], o);
                }
                const bool tied = p.wkind == GDR_GATE_TIED;
                const float de_b = acc[3] + (tied ? acc[2] : 0.f);
                float gsc[3] = {acc[4], kk * de_b, kk * acc[2]};  // dalpha, db, dw for row i
                if (g == 0 && row_ok) {
                    const size_t gi = tok_of(t0 + tau0 + u) * p.dk_ + i;
                    p.dq[gi] = acc[0];
                    p.dk[gi] = acc[1] + bg * acc[3] + wg * acc[2];
                    if (p.akind == GDR_GATE_CHANNEL) p.dalpha[gi] = gsc[0];
                    if (p.bkind == GDR_GATE_CHANNEL) p.db[gi] = gsc[1];
                    if (p.wkind == GDR_GATE_CHANNEL) p.dw[gi] = gsc[2];
                }
                if (p.GP) {  // scalar gates: this warp's rows, summed
                    if (g != 0 || !row_ok)
#pragma unroll
                        for (int qy = 0; qy < 3; ++qy) gsc[qy] = 0.f;
                    for (int o = tpr; o < 32; o <<= 1)
#pragma unroll
                        for (int qy = 0; qy < 3; ++qy) gsc[qy] += __shfl_xor_sync(0xffffffffu, gsc[qy], o);
                    if (lane == 0)
#pragma unroll
                        for (int qy = 0; qy < 3; ++qy) sred[(u * 3 + qy) * (kChunkThreads / 32) + warp] = gsc[qy];
                }
            }
        }
        if (p.GP) {  // the CTA's partial sum per token and scalar gate
            __syncthreads();
            if (tid < kSub * 3) {
                const int u = tid / 3, qy = tid % 3;
                if (u < ns) {
                    float sv = 0.f;
#pragma unroll
                    for (int w = 0; w < kChunkThreads / 32; ++w) sv += sred[(u * 3 + qy) * (kChunkThreads / 32) + w];
                    const size_t BTH = (size_t)p.B * p.T * p.H;
                    p.GP[((size_t)qy * p.nrb + rb) * BTH + tok_of(t0 + tau0 + u)] = sv;
                }
            }
        }
    }
}

// ----------------------------------------------------------------- pass 3 --
__global__ void bwd_gate_sum_kernel(Params p) {
    const size_t BTH = (size_t)p.B * p.T * p.H;
    const size_t n = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    if (n >= BTH) return;
    const int kinds[3] = {p.akind, p.bkind, p.wkind};
    float* dst[3] = {p.dalpha, p.db, p.dw};
#pragma unroll
    for (int qy = 0; qy < 3; ++qy) {
        if (kinds[qy] != GDR_GATE_SCALAR) continue;
        float s = 0.f;
        for (int rb = 0; rb < p.nrb; ++rb) s += p.GP[((size_t)qy * p.nrb + rb) * BTH + n];
        dst[qy][n] = s;
    }
}

// Grouped heads: dq, dk of a q/k head are the sums over the value heads that
// share it (value heads hq G .. hq G + G - 1), added in that order.
__global__ void bwd_group_sum_kernel(Params p) {
    const size_t n = blockIdx.x * (size_t)blockDim.x + threadIdx.x;  // over [B, T, H_qk, d_k]
    const size_t total = (size_t)p.B * p.T * p.Hq * p.dk_;
    if (n >= total) return;
    const int i = (int)(n % p.dk_);
    const size_t tq = n / p.dk_;  // (b t) H_qk + hq
    const size_t bt = tq / p.Hq;
    const int hq = (int)(tq % p.Hq);
    float sq = 0.f, sk = 0.f;
    for (int g = 0; g < p.group; ++g) {
        const size_t src = (bt * p.H + (size_t)hq * p.group + g) * p.dk_ + i;
        sq += p.dq[src];
        sk += p.dk[src];
    }
    p.dq_out[n] = sq;
    p.dk_out[n] = sk;
}

int threads_per_row(int dv) {
    int t = 1;
    while (8 * t < dv) t <<= 1;
    return t;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
    size_t ckS, ckG, R, DR, GP, DQ, DK, FW, total;
};

WsLayout ws_layout(int B, int T, int H, int dk, int dv, bool grouped) {
    WsLayout l{};
    const size_t nch = (size_t)(T + kC - 1) / kC;
    const size_t ck = round256((size_t)B * H * nch * dk * dv * sizeof(float));
    const size_t rr = round256((size_t)B * T * H * dv * sizeof(float));
    const int nrb = (dk + kChunkThreads / threads_per_row(dv) - 1) / (kChunkThreads / threads_per_row(dv));
    const size_t gp = round256((size_t)3 * nrb * B * T * H * sizeof(float));
    l.ckS = 0;
    l.ckG = l.ckS + ck;
    l.R = l.ckG + ck;
    l.DR = l.R + rr;
    l.GP = l.DR + rr;
    const size_t gq = grouped ? round256((size_t)B * T * H * dk * sizeof(float)) : 0;
    l.DQ = l.GP + gp;
    l.DK = l.DQ + gq;
    // d_k = d_v = 128: the forward's per-chunk factors (-W, P), which the
    // tensor-core path computes again to checkpoint S and r on tensor cores
    l.FW = l.DK + gq;
    l.total = l.FW + (dk == 128 && dv == 128 ? round256(twopass_workspace_bytes(B, T, H, dv)) : 0);
    return l;
}

// tc_maps (q, k, v, dO tensor maps) selects the tensor-core path of the Gated
// DeltaNet form: the forward two-pass kernels (their factors in fw, maps
// fw_maps) checkpoint the state at every chunk start and U = beta v - r of
// every token; the chunkwise gradient pass (its factors in the same
// workspace region once the forward is done, maps gw_maps) gives the state
// gradient at every chunk end, dr, dv and dS0; the tensor-core pass 2 writes
// the scalar gate gradients itself. On this path the checkpoints are bf16
// (the start of each checkpoint region; ck_maps: U, dr, S, G, then the fp32
// store maps of dq and dk).
template <typename TI>
cudaError_t launch_typed(Params p, const CUtensorMap* tc_maps, const CUtensorMap* fw_maps, void* fw,
                         const CUtensorMap* gw_maps, const CUtensorMap* ck_maps, cudaStream_t st) {
    cudaError_t e;
    if (tc_maps) {
        e = launch_chunk_twopass_gdn(tc_maps, fw_maps, fw, p.alpha, p.b, p.S0, nullptr, nullptr,
                                     p.d_status, p.B, p.T, p.H, p.dv_, p.group, st,
                                     reinterpret_cast<__nv_bfloat16*>(p.ckS),
                                     reinterpret_cast<__nv_bfloat16*>(p.R));
        if (e != cudaSuccess) return e;
        e = launch_bwd_grad_tc(&tc_maps[0], &tc_maps[1], &tc_maps[3], gw_maps, p.alpha, p.b, p.dST,
                               reinterpret_cast<__nv_bfloat16*>(p.ckG), reinterpret_cast<__nv_bfloat16*>(p.DR),
                               p.dv, p.dS0, p.d_status, p.B, p.T, p.H, p.dv_, p.group, st);
        if (e != cudaSuccess) return e;
        e = launch_bwd_chunk_tc(tc_maps, ck_maps, p.alpha, p.b, p.dq, p.dk, p.dalpha, p.db, p.d_status,
                                p.B, p.T, p.H, p.group, p.nchunks, st);
        if (e != cudaSuccess) return e;
        if (p.group > 1) {
            const size_t n = (size_t)p.B * p.T * p.Hq * p.dk_;
            bwd_group_sum_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(p);
            e = cudaGetLastError();
        }
        return e;
    }
    const dim3 sgrid((p.dv_ + kScanCols * kScanWarps - 1) / (kScanCols * kScanWarps), p.H, 2 * p.B);
    if (p.dk_ > kStagedMaxDK)
        bwd_scan_kernel<TI, 8><<<sgrid, kScanWarps * 32, 0, st>>>(p);
    else if ((p.dk_ * sizeof(TI)) % 16 == 0)
        bwd_scan_staged_kernel<TI><<<sgrid, kScanWarps * 32, 0, st>>>(p);
    else
        bwd_scan_kernel<TI, 4><<<sgrid, kScanWarps * 32, 0, st>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const uint32_t smem = chunk_smem(p.tpr).total;
    void (*kern)(Params) = bwd_chunk_kernel<TI>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(p.nrb, p.nchunks, p.B * p.H), kChunkThreads, smem, st>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.GP) {
        const size_t BTH = (size_t)p.B * p.T * p.H;
        bwd_gate_sum_kernel<<<(unsigned)((BTH + 255) / 256), 256, 0, st>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (p.group > 1) {
        const size_t n = (size_t)p.B * p.T * p.Hq * p.dk_;
        bwd_group_sum_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(p);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace bwd
}  // namespace gdr

namespace {
bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool kind_valid(int kind, bool allow_tied) {
    return kind == GDR_GATE_NONE || kind == GDR_GATE_SCALAR || kind == GDR_GATE_CHANNEL ||
           (allow_tied && kind == GDR_GATE_TIED);
}
// A gate (and its gradient) carries data exactly for the scalar and channel kinds.
bool has_data(int kind) { return kind == GDR_GATE_SCALAR || kind == GDR_GATE_CHANNEL; }
bool ptr_matches(int kind, const void* ptr) { return has_data(kind) ? ptr != nullptr : ptr == nullptr; }
}  // namespace

extern "C" {

size_t gdr_chunk_bwd_grouped_workspace_size(int B, int T, int H_qk, int H, int d_k, int d_v) {
    if (B < 1 || H < 1 || T < 1 || d_k < 1 || d_v < 1 || H_qk < 1 || H % H_qk != 0) return 0;
    return gdr::bwd::ws_layout(B, T, H, d_k, d_v, H_qk != H).total;
}

size_t gdr_chunk_bwd_workspace_size(int B, int T, int H, int d_k, int d_v) {
    return gdr_chunk_bwd_grouped_workspace_size(B, T, H, H, d_k, d_v);
}

gdr_status gdr_chunk_bwd_grouped(const void* q, const void* k, const void* v, const void* alpha,
                                 const void* b, const void* w, int alpha_kind, int b_kind,
                                 int w_kind, const float* S0, const void* dO, const float* dS_T,
                                 float* dq, float* dk, float* dv, float* dalpha, float* db,
                                 float* dw, float* dS0, void* workspace, size_t workspace_bytes,
                                 int B, int T, int H_qk, int H, int d_k, int d_v, int chunk,
                                 int dtype, int* d_status, void* stream) {
    if (B < 1 || H < 1 || T < 0 || d_k < 1 || d_v < 1) return GDR_ERR_INVALID_ARG;
    if (H_qk < 1 || H % H_qk != 0) return GDR_ERR_INVALID_ARG;
    if (dtype != GDR_BF16 && dtype != GDR_FP32) return GDR_ERR_INVALID_ARG;
    if (!kind_valid(alpha_kind, false) || !kind_valid(b_kind, false) || !kind_valid(w_kind, true))
        return GDR_ERR_INVALID_ARG;
    if (w_kind == GDR_GATE_TIED && b_kind == GDR_GATE_NONE) return GDR_ERR_INVALID_ARG;
    if (T > 0 && (!ptr_matches(alpha_kind, alpha) || !ptr_matches(b_kind, b) ||
                  !ptr_matches(w_kind, w)))
        return GDR_ERR_INVALID_ARG;
    if (T > 0 && (!ptr_matches(alpha_kind, dalpha) || !ptr_matches(b_kind, db) ||
                  !ptr_matches(w_kind, dw)))
        return GDR_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !dO || !dq || !dk || !dv)) return GDR_ERR_INVALID_ARG;
    if (chunk != 64) return GDR_ERR_UNSUPPORTED;
    if (d_k > gdr::bwd::kMaxDK || d_v % 8 != 0 || d_v > gdr::bwd::kMaxDV)
        return GDR_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t state_bytes = (size_t)B * H * d_k * d_v * sizeof(float);
    if (T == 0) {  // dS0 = dS_T
        if (!dS0) return GDR_OK;
        cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, state_bytes, cudaMemcpyDeviceToDevice, st)
                             : cudaMemsetAsync(dS0, 0, state_bytes, st);
        return e == cudaSuccess ? GDR_OK : GDR_ERR_LAUNCH;
    }
    const int nch = (T + gdr::bwd::kC - 1) / gdr::bwd::kC;
    if (nch > 65535 || (size_t)B * H > 65535u) return GDR_ERR_UNSUPPORTED;  // grid limits
    // vector rows move in 16-byte pieces; scalar gates and their gradients are
    // read and written one element at a time and need only element alignment
    const void* ptrs[] = {q, k, v, dO, dq, dk, dv, S0, dS_T, dS0};
    for (const void* ptr : ptrs)
        if (ptr && !a16(ptr)) return GDR_ERR_MISALIGNED;
    const int kinds[3] = {alpha_kind, b_kind, w_kind};
    const void* gates[3] = {alpha, b, w};
    const void* grads[3] = {dalpha, db, dw};
    for (int i = 0; i < 3; ++i)
        if (kinds[i] == GDR_GATE_CHANNEL && (!a16(gates[i]) || (grads[i] && !a16(grads[i]))))
            return GDR_ERR_MISALIGNED;
    const bool grouped = H_qk != H;
    const gdr::bwd::WsLayout wl = gdr::bwd::ws_layout(B, T, H, d_k, d_v, grouped);
    if (!workspace || workspace_bytes < wl.total) return GDR_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDR_ERR_MISALIGNED;

    unsigned char* ws = static_cast<unsigned char*>(workspace);
    gdr::bwd::Params p;
    p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.b = b; p.w = w; p.dO = dO;
    p.S0 = S0; p.dST = dS_T;
    p.dv = dv; p.dalpha = dalpha; p.db = db; p.dw = dw; p.dS0 = dS0;
    if (grouped) {  // per-value-head dq, dk in the workspace, summed over each group at the end
        p.dq = reinterpret_cast<float*>(ws + wl.DQ);
        p.dk = reinterpret_cast<float*>(ws + wl.DK);
        p.dq_out = dq;
        p.dk_out = dk;
    } else {
        p.dq = dq;
        p.dk = dk;
        p.dq_out = p.dk_out = nullptr;
    }
    p.ckS = reinterpret_cast<float*>(ws + wl.ckS);
    p.ckG = reinterpret_cast<float*>(ws + wl.ckG);
    p.R = reinterpret_cast<float*>(ws + wl.R);
    p.DR = reinterpret_cast<float*>(ws + wl.DR);
    const bool any_scalar = alpha_kind == GDR_GATE_SCALAR || b_kind == GDR_GATE_SCALAR ||
                            w_kind == GDR_GATE_SCALAR;
    p.GP = any_scalar ? reinterpret_cast<float*>(ws + wl.GP) : nullptr;
    p.B = B; p.T = T; p.H = H; p.Hq = H_qk; p.group = H / H_qk; p.dk_ = d_k; p.dv_ = d_v;
    p.akind = alpha_kind; p.bkind = b_kind; p.wkind = w_kind;
    p.nchunks = nch;
    p.tpr = gdr::bwd::threads_per_row(d_v);
    const int RB = gdr::bwd::kChunkThreads / p.tpr;
    p.nrb = (d_k + RB - 1) / RB;
    p.d_status = d_status;
    // the Gated DeltaNet form on tensor cores: scalar decay, tied scalar beta,
    // bf16, d_k = d_v = 128
    CUtensorMap maps[4], fw_maps[3], gw_maps[3], ck_maps[6];
    const CUtensorMap* tc_maps = nullptr;
    void* fw = ws + wl.FW;
    // the checkpoints' tensor maps view each as [B H nchunks 128, 128] rows (int32 coordinates)
    const bool ck_rows_fit = (size_t)B * H * nch * 128 <= (size_t)INT32_MAX;
    if (dtype == GDR_BF16 && d_k == 128 && d_v == 128 && alpha_kind == GDR_GATE_SCALAR &&
        b_kind == GDR_GATE_SCALAR && w_kind == GDR_GATE_TIED && ck_rows_fit) {
        const int ck_rows = B * H * nch * 128;
        if (!gdr::make_tma_map_bf16(&maps[0], q, B, T, H_qk, d_k) ||
            !gdr::make_tma_map_bf16(&maps[1], k, B, T, H_qk, d_k) ||
            !gdr::make_tma_map_bf16(&maps[2], v, B, T, H, d_v) ||
            !gdr::make_tma_map_bf16(&maps[3], dO, B, T, H, d_v) ||
            !gdr::make_tma_map_bf16(&fw_maps[0], fw, B, T, H, d_k) ||
            !gdr::make_tma_map_bf16(&fw_maps[1], ws + wl.FW + (size_t)B * T * H * d_k * 2, B, T, H, d_v) ||
            !gdr::make_tma_map_bf16(&fw_maps[2], ws + wl.FW + (size_t)B * T * H * (d_k + d_v) * 2, B, T, H, 64) ||
            // the gradient pass's factors X, Aq T, Diag(g) Q take the same region
            // (2 B T H (128 + 64 + 128) bytes) once the forward has read its own
            !gdr::make_tma_map_bf16(&gw_maps[0], fw, B, T, H, d_k) ||
            !gdr::make_tma_map_bf16(&gw_maps[1], ws + wl.FW + (size_t)B * T * H * d_k * 2, B, T, H, 64) ||
            !gdr::make_tma_map_bf16(&gw_maps[2], ws + wl.FW + (size_t)B * T * H * (d_k + 64) * 2, B, T, H, d_k) ||
            // bf16 checkpoints: U, dr per token; S, G per chunk
            !gdr::make_tma_map_bf16(&ck_maps[0], ws + wl.R, B, T, H, d_v) ||
            !gdr::make_tma_map_bf16(&ck_maps[1], ws + wl.DR, B, T, H, d_v) ||
            !gdr::make_tma_map_bf16(&ck_maps[2], ws + wl.ckS, 1, ck_rows, 1, d_v) ||
            !gdr::make_tma_map_bf16(&ck_maps[3], ws + wl.ckG, 1, ck_rows, 1, d_v) ||
            !gdr::make_tma_map_f32(&ck_maps[4], p.dq, B, T, H, d_k) ||
            !gdr::make_tma_map_f32(&ck_maps[5], p.dk, B, T, H, d_k))
            return GDR_ERR_NO_DEVICE;
        tc_maps = maps;
        p.GP = nullptr;
    }
    const cudaError_t e = dtype == GDR_BF16
                              ? gdr::bwd::launch_typed<__nv_bfloat16>(p, tc_maps, fw_maps, fw, gw_maps, ck_maps, st)
                              : gdr::bwd::launch_typed<float>(p, nullptr, nullptr, nullptr, nullptr, nullptr, st);
    return e == cudaSuccess ? GDR_OK : GDR_ERR_LAUNCH;
}

gdr_status gdr_chunk_bwd(const void* q, const void* k, const void* v, const void* alpha,
                         const void* b, const void* w, int alpha_kind, int b_kind, int w_kind,
                         const float* S0, const void* dO, const float* dS_T, float* dq, float* dk,
                         float* dv, float* dalpha, float* db, float* dw, float* dS0,
                         void* workspace, size_t workspace_bytes, int B, int T, int H, int d_k,
                         int d_v, int chunk, int dtype, int* d_status, void* stream) {
    return gdr_chunk_bwd_grouped(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S0, dO, dS_T,
                                 dq, dk, dv, dalpha, db, dw, dS0, workspace, workspace_bytes, B, T,
                                 H, H, d_k, d_v, chunk, dtype, d_status, stream);
}

}  // extern "C"
