// Backward pass of the gated delta rule: fp32 arithmetic on CUDA cores, one
// thread-block cluster per head.
//
// The pages ask for a gate-aware backward pass ("Erase-then-Delta Attention"
// (Gated DeltaNet-2), abstract) without printing one. This is reverse-mode
// differentiation of the token recurrence
//   S' = Diag(alpha_t) S_{t-1},  r_t = (b_t . k_t) S',
//   S_t = S' - k_t^T r_t + (w_t . k_t)^T v_t,  o_t = q_t S_t
// ("Recurrent Memory: Write, Erase, Decay, Read", sections 01-05), run from the
// last token to the first with G = dL/dS_t (e = b.k, u = w.k):
//   dq_t = dO_t S_t^T,   G += q_t^T dO_t,
//   dv_t = u G,  du = G v_t^T,  dk = -G r_t^T,  dr = -k G,
//   de = S' dr^T,  dS' = G + e^T dr,  dalpha = rowsum(dS' . S_{t-1}),
//   G <- Diag(alpha_t) dS',  dk += b.de + w.du,  db = k.de,  dw = k.du.
//
// Launches:
//  1. bwd_ckpt_kernel: the forward recurrence, storing the state at the start
//     of every 64-token chunk in the caller's workspace.
//  2. bwd_main_kernel: chunks last to first. Per chunk the forward is
//     recomputed from its checkpoint, keeping r_t of every token and the state
//     at every 8-token sub-chunk start in shared memory; then, per sub-chunk
//     last to first, its 8 states are rebuilt in registers (no reduction
//     needed once r_t is known) and the reverse step runs token by token.
// Layout: the cluster's CTA x owns state columns [16x, 16x + 16) of one head;
// warp w of its 8 holds rows 32 (w % 4) + lane and columns 8 (w / 4) .. + 8 of
// that slice, so S and G are 8 + 8 fp32 registers per thread. Sums over rows
// (r, dr, dv) stay inside the CTA (warp shuffles, then four warps through
// shared memory); sums over columns (the dq, dk, du, de, dalpha rows) are
// partial per CTA and are added across the cluster through distributed shared
// memory once per sub-chunk.
#include "common.cuh"

namespace gdr {
namespace bwd {

constexpr int kC = 64;               // checkpoint interval (the chunk)
constexpr int kSub = 8;              // sub-chunk: states rebuilt in registers
constexpr int kNSub = kC / kSub;
constexpr int kNC = 16;              // state columns per CTA
constexpr int kThreads = 256;
constexpr int kRows = 128;           // d_k limit (one thread per row and column half)
constexpr int kMaxNB = 8;            // portable cluster size: d_v <= 128
constexpr int kQty = 5;              // per-row partials: dq, dk (from r), du, de, dalpha

struct Params {
    const void *q, *k, *v, *alpha, *b, *w, *dO;
    const float *S0, *dST;
    float *dq, *dk, *dv, *dalpha, *db, *dw, *dS0, *ckpt;
    int T, H, dk_, dv_, akind, bkind, wkind, nchunks;
};

template <typename TI>
__device__ __forceinline__ float ld1(const void* p, size_t i) {
    return to_f32(static_cast<const TI*>(p)[i]);
}

// Eight consecutive elements (16- or 32-byte aligned) widened to fp32.
template <typename TI>
__device__ __forceinline__ void load8(const void* p, size_t off, float (&x)[8]);
template <>
__device__ __forceinline__ void load8<float>(const void* p, size_t off, float (&x)[8]) {
    const float4* s = reinterpret_cast<const float4*>(static_cast<const float*>(p) + off);
    const float4 a = s[0], b = s[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const void* p, size_t off, float (&x)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p) + off);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        x[2 * c] = __uint_as_float(w[c] << 16);
        x[2 * c + 1] = __uint_as_float(w[c] & 0xffff0000u);
    }
}

// Per-row scalars of one token for key channel i (neutral beyond d_k).
struct Row {
    float q, k, a, bg, wg;
};

template <typename TI>
__device__ __forceinline__ Row load_row(const Params& p, size_t tok, int i) {
    Row r{0.f, 0.f, 1.f, 0.f, 0.f};
    if (i < p.dk_) {
        const size_t gi = tok * p.dk_ + i;
        r.q = ld1<TI>(p.q, gi);
        r.k = ld1<TI>(p.k, gi);
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

// Sum over the warp's 32 lanes of NV values per lane, scattered: on return
// the lane holds the total of value (lane / (32 / NV)). Each halving step
// sends the half of the values the partner keeps.
template <int NV>
__device__ __forceinline__ float warp_reduce_scatter(float* x, int lane) {
    int off = 16;
#pragma unroll
    for (int half = NV / 2; half >= 1; half >>= 1, off >>= 1) {
        const bool hi = (lane & off) != 0;
#pragma unroll
        for (int v = 0; v < half; ++v) {
            const float send = hi ? x[v] : x[v + half];
            const float keep = hi ? x[v + half] : x[v];
            x[v] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    float s = x[0];
#pragma unroll
    for (; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return s;
}

// Row-group partial sums: red[parity][column half][row group][16].
__device__ __forceinline__ float* red_at(float* red, int par, int cg, int rg) {
    return red + ((par * 2 + cg) * 4 + rg) * 16;
}

// Column sums over the CTA's 128 rows of x[0..NV): warp shuffles, then one
// barrier; the four row-group totals are read back with red_sum8.
template <int NV>
__device__ __forceinline__ void colsum_publish(float* x, float* red, int par, int cg, int rg,
                                               int lane) {
    const float s = warp_reduce_scatter<NV>(x, lane);
    constexpr int G = 32 / NV;
    if ((lane & (G - 1)) == 0) red_at(red, par, cg, rg)[lane / G] = s;
    __syncthreads();
}

__device__ __forceinline__ void red_sum8(const float* red, int par, int cg, int c0, float (&out)[8]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) out[c] = 0.f;
#pragma unroll
    for (int rg = 0; rg < 4; ++rg) {
        const float4* s = reinterpret_cast<const float4*>(red_at(const_cast<float*>(red), par, cg, rg) + c0);
        const float4 a = s[0], b = s[1];
        out[0] += a.x; out[1] += a.y; out[2] += a.z; out[3] += a.w;
        out[4] += b.x; out[5] += b.y; out[6] += b.z; out[7] += b.w;
    }
}

// One forward token: S <- Diag(a) S; r = (b.k) S (column sums); S <- S - k^T r + (w.k)^T v.
__device__ __forceinline__ void fwd_step(float (&S)[8], const Row& rw, const float (&v)[8], float* red,
                                         int par, int cg, int rg, int lane, float (&r)[8]) {
    const float e = rw.bg * rw.k, u = rw.wg * rw.k;
    float x[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        S[c] *= rw.a;
        x[c] = e * S[c];
    }
    colsum_publish<8>(x, red, par, cg, rg, lane);
    red_sum8(red, par, cg, 0, r);
#pragma unroll
    for (int c = 0; c < 8; ++c) S[c] = fmaf(-rw.k, r[c], fmaf(u, v[c], S[c]));
}

__device__ __forceinline__ void store8(float* dst, const float (&x)[8]) {
    reinterpret_cast<float4*>(dst)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(dst)[1] = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ void load8f(const float* src, float (&x)[8]) {
    const float4 a = reinterpret_cast<const float4*>(src)[0];
    const float4 b = reinterpret_cast<const float4*>(src)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// ----------------------------------------------------------------- pass 1 --
template <typename TI>
__global__ void __launch_bounds__(kThreads) bwd_ckpt_kernel(Params p) {
    __shared__ __align__(16) float red[2 * 2 * 4 * 16];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, rg = warp & 3, cg = warp >> 2;
    const int i = 32 * rg + lane;
    const int b = blockIdx.z, h = blockIdx.y;
    const int col = kNC * blockIdx.x + 8 * cg;
    const size_t head = (size_t)b * p.H + h;
    const bool row_ok = i < p.dk_;
    float S[8];
    if (p.S0 && row_ok) load8f(p.S0 + (head * p.dk_ + i) * p.dv_ + col, S);
    else
        for (int c = 0; c < 8; ++c) S[c] = 0.f;
    auto tok_of = [&](int t) { return ((size_t)b * p.T + t) * p.H + h; };
    Row nr = load_row<TI>(p, tok_of(0), i);
    float nv[8];
    load8<TI>(p.v, tok_of(0) * p.dv_ + col, nv);
    int par = 0;
    for (int t = 0; t < p.T; ++t) {
        const Row rw = nr;
        float v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) v[c] = nv[c];
        if (t + 1 < p.T) {  // next token's inputs are in flight during this step
            nr = load_row<TI>(p, tok_of(t + 1), i);
            load8<TI>(p.v, tok_of(t + 1) * p.dv_ + col, nv);
        }
        if (t % kC == 0 && row_ok)
            store8(p.ckpt + (((head * p.nchunks + t / kC) * p.dk_) + i) * p.dv_ + col, S);
        float r[8];
        fwd_step(S, rw, v, red, par, cg, rg, lane, r);
        par ^= 1;
    }
}

// ----------------------------------------------------------------- pass 2 --
struct __align__(16) MainSmem {
    float4 subck[kNSub][2][2][kRows];     // state at sub-chunk starts: [sub][col half][float4][row]
    float rch[kC][kNC];                   // r_t of every token of the chunk
    float red[2 * 2 * 4 * 16];            // row-group partial sums
    float part[2][kSub][kQty][2][kRows];  // per-row partials: [buffer][token][qty][col half][row]
    float sred[kSub][3][4];               // scalar-gate totals: [token][gate][warp]
};

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile(
        "barrier.cluster.arrive.release.aligned;\n\t"
        "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t map_to_rank(uint32_t local_smem, int rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_smem), "r"(rank));
    return r;
}

__device__ __forceinline__ float ld_cluster(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

template <typename TI>
__global__ void __launch_bounds__(kThreads, 1) bwd_main_kernel(Params p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    MainSmem& sm = *reinterpret_cast<MainSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, rg = warp & 3, cg = warp >> 2;
    const int i = 32 * rg + lane;
    const int rank = blockIdx.x, NB = gridDim.x;  // the cluster spans gridDim.x
    const int b = blockIdx.z, h = blockIdx.y;
    const int col = kNC * rank + 8 * cg;
    const size_t head = (size_t)b * p.H + h;
    const bool row_ok = i < p.dk_;
    auto tok_of = [&](int t) { return ((size_t)b * p.T + t) * p.H + h; };

    float G[8];
    if (p.dST && row_ok) load8f(p.dST + (head * p.dk_ + i) * p.dv_ + col, G);
    else
        for (int c = 0; c < 8; ++c) G[c] = 0.f;

    const uint32_t part_local = smem_u32(&sm.part[0][0][0][0][0]);
    int par = 0, sbuf = 0;
    for (int c = p.nchunks - 1; c >= 0; --c) {
        const int t0 = c * kC;
        const int L = min(kC, p.T - t0);
        // ---- forward over the chunk from its checkpoint: r_t, sub-chunk states
        float S[8];
        if (row_ok) load8f(p.ckpt + (((head * p.nchunks + c) * p.dk_) + i) * p.dv_ + col, S);
        else
            for (int cc = 0; cc < 8; ++cc) S[cc] = 0.f;
        Row nr = load_row<TI>(p, tok_of(t0), i);
        float nv[8];
        load8<TI>(p.v, tok_of(t0) * p.dv_ + col, nv);
        for (int tau = 0; tau < L; ++tau) {
            const Row rw = nr;
            float v[8];
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) v[cc] = nv[cc];
            if (tau + 1 < L) {
                nr = load_row<TI>(p, tok_of(t0 + tau + 1), i);
                load8<TI>(p.v, tok_of(t0 + tau + 1) * p.dv_ + col, nv);
            }
            if (tau % kSub == 0) {
                sm.subck[tau / kSub][cg][0][i] = make_float4(S[0], S[1], S[2], S[3]);
                sm.subck[tau / kSub][cg][1][i] = make_float4(S[4], S[5], S[6], S[7]);
            }
            float r[8];
            fwd_step(S, rw, v, sm.red, par, cg, rg, lane, r);
            par ^= 1;
            if (rg == 0 && lane == 0) store8(&sm.rch[tau][8 * cg], r);
        }
        __syncthreads();  // rch complete

        // ---- reverse, one sub-chunk at a time
        const int nsub = (L + kSub - 1) / kSub;
        for (int s = nsub - 1; s >= 0; --s) {
            const int tau0 = s * kSub;
            const int ns = min(kSub, L - tau0);
            float Sst[kSub][8];  // S_{t-1} of each token of the sub-chunk
            {
                const float4 a0 = sm.subck[s][cg][0][i], a1 = sm.subck[s][cg][1][i];
                S[0] = a0.x; S[1] = a0.y; S[2] = a0.z; S[3] = a0.w;
                S[4] = a1.x; S[5] = a1.y; S[6] = a1.z; S[7] = a1.w;
            }
#pragma unroll
            for (int u = 0; u < kSub; ++u) {
                if (u < ns) {
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) Sst[u][cc] = S[cc];
                    if (u + 1 < ns) {
                        const size_t tok = tok_of(t0 + tau0 + u);
                        const Row rw = load_row<TI>(p, tok, i);
                        float v[8], r[8];
                        load8<TI>(p.v, tok * p.dv_ + col, v);
                        load8f(&sm.rch[tau0 + u][8 * cg], r);
                        const float uu = rw.wg * rw.k;
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc)
                            S[cc] = fmaf(-rw.k, r[cc], fmaf(uu, v[cc], rw.a * S[cc]));
                    }
                }
            }
#pragma unroll
            for (int u = kSub - 1; u >= 0; --u) {
                if (u < ns) {
                    const size_t tok = tok_of(t0 + tau0 + u);
                    const Row rw = load_row<TI>(p, tok, i);
                    float v[8], d[8], r[8];
                    load8<TI>(p.v, tok * p.dv_ + col, v);
                    load8<TI>(p.dO, tok * p.dv_ + col, d);
                    load8f(&sm.rch[tau0 + u][8 * cg], r);
                    const float e = rw.bg * rw.k, uu = rw.wg * rw.k;
                    // o_t = q_t S_t
                    float pdq = 0.f;
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        const float st = fmaf(-rw.k, r[cc], fmaf(uu, v[cc], rw.a * Sst[u][cc]));
                        pdq = fmaf(st, d[cc], pdq);
                        G[cc] = fmaf(rw.q, d[cc], G[cc]);
                    }
                    // S_t = S' - k^T r + u^T v
                    float x[16], pdu = 0.f, pdkd = 0.f;
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        x[cc] = uu * G[cc];
                        x[8 + cc] = rw.k * G[cc];
                        pdu = fmaf(G[cc], v[cc], pdu);
                        pdkd = fmaf(-G[cc], r[cc], pdkd);
                    }
                    colsum_publish<16>(x, sm.red, par, cg, rg, lane);
                    if (rg == 0 && lane < 8) {
                        float sv = 0.f;
#pragma unroll
                        for (int g = 0; g < 4; ++g) sv += red_at(sm.red, par, cg, g)[lane];
                        p.dv[tok * p.dv_ + col + lane] = sv;
                    }
                    float dr[8];
                    red_sum8(sm.red, par, cg, 8, dr);
                    par ^= 1;
                    // r = e S';  S' = Diag(a) S_{t-1}
                    float pde = 0.f, pdal = 0.f;
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        const float drc = -dr[cc];
                        pde = fmaf(rw.a * Sst[u][cc], drc, pde);
                        const float dsd = fmaf(e, drc, G[cc]);
                        pdal = fmaf(dsd, Sst[u][cc], pdal);
                        G[cc] = rw.a * dsd;
                    }
                    float* pp = &sm.part[sbuf][u][0][cg][i];
                    pp[0] = pdq;
                    pp[2 * kRows] = pdkd;
                    pp[4 * kRows] = pdu;
                    pp[6 * kRows] = pde;
                    pp[8 * kRows] = pdal;
                }
            }
            cluster_sync_all();  // this sub-chunk's partials are visible cluster-wide

            // ---- totals over the cluster: CTA `rank` finishes tokens rank, rank + NB, ...
            if (tid < kRows) {
                for (int u = rank; u < ns; u += NB) {
                    float tot[kQty] = {0.f, 0.f, 0.f, 0.f, 0.f};
                    for (int rk = 0; rk < NB; ++rk) {
                        const uint32_t base = map_to_rank(part_local, rk);
#pragma unroll
                        for (int qy = 0; qy < kQty; ++qy)
#pragma unroll
                            for (int hc = 0; hc < 2; ++hc) {
                                const uint32_t off =
                                    ((((sbuf * kSub + u) * kQty + qy) * 2 + hc) * kRows + tid) * 4u;
                                tot[qy] += ld_cluster(base + off);
                            }
                    }
                    const size_t tok = tok_of(t0 + tau0 + u);
                    const Row rw = load_row<TI>(p, tok, tid);
                    const bool tied = p.wkind == GDR_GATE_TIED;
                    const float de_b = tot[3] + (tied ? tot[2] : 0.f);  // dL/db through e (and u if tied)
                    const float g_a = tot[4], g_b = rw.k * de_b, g_w = rw.k * tot[2];
                    if (tid < p.dk_) {
                        const size_t gi = tok * p.dk_ + tid;
                        p.dq[gi] = tot[0];
                        p.dk[gi] = tot[1] + rw.bg * tot[3] + rw.wg * tot[2];
                        if (p.akind == GDR_GATE_CHANNEL) p.dalpha[gi] = g_a;
                        if (p.bkind == GDR_GATE_CHANNEL) p.db[gi] = g_b;
                        if (p.wkind == GDR_GATE_CHANNEL) p.dw[gi] = g_w;
                    }
                    // scalar gates: sum over the key channels (rows beyond d_k hold zeros)
                    float sc[3] = {g_a, g_b, g_w};
#pragma unroll
                    for (int g = 0; g < 3; ++g)
#pragma unroll
                        for (int o = 16; o >= 1; o >>= 1)
                            sc[g] += __shfl_xor_sync(0xffffffffu, sc[g], o);
                    if (lane == 0)
#pragma unroll
                        for (int g = 0; g < 3; ++g) sm.sred[u][g][warp] = sc[g];
                }
            }
            __syncthreads();
            if (tid < kSub * 3) {
                const int u = tid / 3, g = tid % 3;
                const int kind = g == 0 ? p.akind : g == 1 ? p.bkind : p.wkind;
                if (u < ns && u % NB == rank && kind == GDR_GATE_SCALAR) {
                    const float sv = sm.sred[u][g][0] + sm.sred[u][g][1] + sm.sred[u][g][2] +
                                     sm.sred[u][g][3];
                    float* dst = g == 0 ? p.dalpha : g == 1 ? p.db : p.dw;
                    dst[tok_of(t0 + tau0 + u)] = sv;
                }
            }
            sbuf ^= 1;
        }
        __syncthreads();  // rch and subck are rewritten by the next chunk
    }
    if (p.dS0 && row_ok) store8(p.dS0 + (head * p.dk_ + i) * p.dv_ + col, G);
    cluster_sync_all();  // no CTA leaves while a peer may still read its partials
}

size_t ckpt_bytes(int B, int T, int H, int dk, int dv) {
    if (T <= 0) return 0;
    const size_t nch = (size_t)(T + kC - 1) / kC;
    return (size_t)B * H * nch * dk * dv * sizeof(float);
}

template <typename TI>
cudaError_t launch_typed(const Params& p, int B, int H, cudaStream_t st) {
    const int NB = p.dv_ / kNC;
    bwd_ckpt_kernel<TI><<<dim3(NB, H, B), kThreads, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = sizeof(MainSmem);
    e = cudaFuncSetAttribute(bwd_main_kernel<TI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(NB, H, B);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = NB;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, bwd_main_kernel<TI>, p);
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

size_t gdr_chunk_bwd_workspace_size(int B, int T, int H, int d_k, int d_v) {
    if (B < 1 || H < 1 || T < 1 || d_k < 1 || d_v < 1) return 0;
    return gdr::bwd::ckpt_bytes(B, T, H, d_k, d_v);
}

gdr_status gdr_chunk_bwd(const void* q, const void* k, const void* v, const void* alpha,
                         const void* b, const void* w, int alpha_kind, int b_kind, int w_kind,
                         const float* S0, const void* dO, const float* dS_T, float* dq, float* dk,
                         float* dv, float* dalpha, float* db, float* dw, float* dS0,
                         void* workspace, size_t workspace_bytes, int B, int T, int H, int d_k,
                         int d_v, int chunk, int dtype, int* d_status, void* stream) {
    (void)d_status;  // this path has no bounded waits to report
    if (B < 1 || H < 1 || T < 0 || d_k < 1 || d_v < 1) return GDR_ERR_INVALID_ARG;
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
    if (d_k > gdr::bwd::kRows || d_v % gdr::bwd::kNC != 0 ||
        d_v > gdr::bwd::kNC * gdr::bwd::kMaxNB)
        return GDR_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t state_bytes = (size_t)B * H * d_k * d_v * sizeof(float);
    if (T == 0) {  // dS0 = dS_T
        if (!dS0) return GDR_OK;
        cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, state_bytes, cudaMemcpyDeviceToDevice, st)
                             : cudaMemsetAsync(dS0, 0, state_bytes, st);
        return e == cudaSuccess ? GDR_OK : GDR_ERR_LAUNCH;
    }
    const void* ptrs[] = {q, k, v, dO, dq, dk, dv, S0, dS_T, dS0, dalpha, db, dw, alpha, b, w};
    for (const void* p : ptrs)
        if (p && !a16(p)) return GDR_ERR_MISALIGNED;
    if (!workspace || workspace_bytes < gdr_chunk_bwd_workspace_size(B, T, H, d_k, d_v))
        return GDR_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDR_ERR_MISALIGNED;

    gdr::bwd::Params p;
    p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.b = b; p.w = w; p.dO = dO;
    p.S0 = S0; p.dST = dS_T;
    p.dq = dq; p.dk = dk; p.dv = dv; p.dalpha = dalpha; p.db = db; p.dw = dw; p.dS0 = dS0;
    p.ckpt = static_cast<float*>(workspace);
    p.T = T; p.H = H; p.dk_ = d_k; p.dv_ = d_v;
    p.akind = alpha_kind; p.bkind = b_kind; p.wkind = w_kind;
    p.nchunks = (T + gdr::bwd::kC - 1) / gdr::bwd::kC;
    const cudaError_t e = dtype == GDR_BF16 ? gdr::bwd::launch_typed<__nv_bfloat16>(p, B, H, st)
                                            : gdr::bwd::launch_typed<float>(p, B, H, st);
    return e == cudaSuccess ? GDR_OK : GDR_ERR_LAUNCH;
}

}  // extern "C"
