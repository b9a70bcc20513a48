// Two-pass chunkwise forward for the Gated DeltaNet form (scalar decay per
// token, tied scalar b = w = beta) on sm_100a tensor cores.
//
// The per-chunk WY/UT factors depend only on the chunk's own keys, values and
// gates, not on the state ("Erase-then-Delta Attention" abstract: chunkwise
// WY form with the decay absorbed into the erase factors; "Recurrent Memory:
// Write, Erase, Decay, Read" section 03 for the chunk reassociation). So the
// forward runs in two passes:
//
//   pass 1 (prep, persistent CTAs over all chunks of all heads):
//     A  = Diag(beta) ((K K^T) . G) strict lower, G_rj = g_r / g_j
//     T  = (I + A)^-1
//     -W = -T Diag(beta g) K                        -> workspace [B,T,H,128] bf16
//     P  =  T Diag(beta) V                          -> workspace [B,T,H,d_v] bf16
//   pass 2 (state, one CTA per (batch, head, 64 columns of d_v), chunks in order):
//     U  = P - W S                                  (MMA [Q ; -W] S, plus P)
//     Aq = (Q K^T) . G                              lower, incl. the diagonal
//     O  = Diag(g) (Q S) + Aq U
//     S' = g_{n-1} S + (Diag(g_{n-1}/g) K)^T U
// with l_r the prefix sum of log2 alpha over the chunk and g_r = 2^l_r. The
// scalar decay factors out of every product, so each ratio g_r / g_j =
// 2^(l_r - l_j) (r >= j) is formed per element on the accumulator unload:
// every factor is at most 1 and no alpha in (0, 1] leaves the range.
//
// Pass 2's per-chunk chain is two MMA round trips; the triangular solve and
// the W / P products (most of the single-pass kernel's chain) run in pass 1
// with every chunk of every head in flight at once.
#include "chunk_common.cuh"

namespace gdr {
namespace twopass {

using namespace chunkc;

// Optional phase tracing (build with -DGDR_TRACE_PHASES): clock64() stamps of
// thread 0 at phase boundaries, pass 1 for the first 64 items of CTA 0 (slots
// 0..7 of row it), pass 2 for the first 64 chunks of CTA (0, 0, 0) (slots
// 8..15). gdr_trace_twopass_read() copies them out.
#ifdef GDR_TRACE_PHASES
__device__ unsigned long long g_trace2[64 * 16];
#define GDR_TRACE_P(k)                                                                     \
    do {                                                                                  \
        if (blockIdx.x == 0 && threadIdx.x == 0 && it < 64)                               \
            g_trace2[it * 16 + (k)] = clock64();                                          \
    } while (0)
#define GDR_TRACE_S(k, thr)                                                                \
    do {                                                                                  \
        if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == (thr) && \
            ci < 64)                                                                      \
            g_trace2[ci * 16 + 8 + (k)] = clock64();                                      \
    } while (0)
#else
#define GDR_TRACE_P(k) \
    do {              \
    } while (0)
#define GDR_TRACE_S(k, thr) \
    do {                   \
    } while (0)
#endif

// ---- pass 1 shared memory (bytes from a 1024-aligned base) ----------------
// Persistent CTAs (two per SM) walk the (chunk, head, batch) items; each
// item's K / V tiles are loaded while the previous item is computed, and -W
// and P leave through shared-memory staging tiles and TMA bulk stores.
// M = 128 MMAs read A rows 64..127 beyond each 64-row operand; those rows
// land in the next region (garbage rows whose outputs are never read).
constexpr uint32_t P_OFF_K = 0;        // K [64 x 128] bf16, two 8 KB column halves; 2 buffers
constexpr uint32_t P_OFF_Q = 32768;    // Q [64 x 128] bf16 (one buffer); then the Aq staging tile
constexpr uint32_t P_OFF_V = 49152;    // V [64 x d_v] bf16, d_v / 64 tiles of 8 KB (one buffer)
constexpr uint32_t P_OFF_A32 = 65536;  // A fp32 [64 x 64]; then L, PRE bf16; then -W staging
constexpr uint32_t P_OFF_T32 = 81920;  // T fp32 [64 x 64]; then P staging
constexpr uint32_t P_OFF_SCR = 98304;  // solve scratch fp32 (5 KB)
constexpr uint32_t P_OFF_SMALL = 103424;
constexpr uint32_t P_SMEM_BYTES = P_OFF_SMALL + 2048 + 1024;
constexpr uint32_t P_TM_D1 = 0, P_TM_DQ = 64, P_TM_D3 = 0, P_TM_D2 = 128, P_TM_COLS = 256;

struct PrepParams {
    const void* alpha;
    const void* beta;
    int* d_status;
    int T, H, dv, nitems;
    int group;  // value heads per k head (k read at head h / group)
};

// Loads: K two items ahead (two buffers), Q once the current item's Q K^T has
// read it and its Aq store has left the tile, V once the current item's P
// product has read it. Q K^T rides in the otherwise unused TMEM lanes 64..127
// of the K K^T batch (its operand starts 8 KB before Q), so the warps that own
// those lanes form Aq while the others form A.
__global__ void __launch_bounds__(NT, 2) prep_gdn_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                         const __grid_constant__ CUtensorMap tm_k,
                                                         const __grid_constant__ CUtensorMap tm_v,
                                                         const __grid_constant__ CUtensorMap tm_wout,
                                                         const __grid_constant__ CUtensorMap tm_pout,
                                                         const __grid_constant__ CUtensorMap tm_aqout,
                                                         const PrepParams pp) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, wg = warp >> 2, row = tid & 127;
    const int T = pp.T, H = pp.H, dv = pp.dv;
    const int nchunks = (T + C - 1) / C;
    const int nvt = dv / 64;

    float* s_beta = reinterpret_cast<float*>(sm + P_OFF_SMALL);
    float* s_l = s_beta + 64;   // log2 prefix of alpha over the chunk
    float* s_g = s_beta + 192;
    float* s_alpha = s_beta + 256;
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + P_OFF_SMALL + 1280);  // [2]: K
    uint64_t* bar_mma = bar_tma + 2;
    uint64_t* bar_q = bar_tma + 3;
    uint64_t* bar_v = bar_tma + 4;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + P_OFF_SMALL + 1328);
    const uint32_t sbase = smem_u32(sm);

    auto coords = [&](int item, int& ci, int& h, int& bb) {
        ci = item % nchunks;
        const int hb = item / nchunks;
        h = hb % H;
        bb = hb / H;
    };
    auto issue_k = [&](int item, int buf) {
        int ci, h, bb;
        coords(item, ci, h, bb);
        const int hq = h / pp.group;
        mbar_expect_tx(&bar_tma[buf], 2u * 8192u);
        tma_load_4d(sm + P_OFF_K + buf * 16384, &tm_k, &bar_tma[buf], 0, hq, ci * C, bb);
        tma_load_4d(sm + P_OFF_K + buf * 16384 + 8192, &tm_k, &bar_tma[buf], 64, hq, ci * C, bb);
    };
    auto issue_q = [&](int item) {
        int ci, h, bb;
        coords(item, ci, h, bb);
        const int hq = h / pp.group;
        mbar_expect_tx(bar_q, 2u * 8192u);
        tma_load_4d(sm + P_OFF_Q, &tm_q, bar_q, 0, hq, ci * C, bb);
        tma_load_4d(sm + P_OFF_Q + 8192, &tm_q, bar_q, 64, hq, ci * C, bb);
    };
    auto issue_v = [&](int item) {
        int ci, h, bb;
        coords(item, ci, h, bb);
        mbar_expect_tx(bar_v, (uint32_t)nvt * 8192u);
        for (int vt = 0; vt < nvt; ++vt)
            tma_load_4d(sm + P_OFF_V + vt * 8192, &tm_v, bar_v, vt * 64, h, ci * C, bb);
    };
    unsigned short g_a = 0, g_b = 0;
    auto load_gates = [&](int item) {
        if (tid < C) {
            int ci, h, bb;
            coords(item, ci, h, bb);
            const int t = min(ci * C + tid, T - 1);
            const size_t gi = ((size_t)bb * T + t) * H + h;
            g_a = reinterpret_cast<const unsigned short*>(pp.alpha)[gi];
            g_b = reinterpret_cast<const unsigned short*>(pp.beta)[gi];
        }
    };
    auto bits_to_f32 = [](unsigned short u) { return __uint_as_float((uint32_t)u << 16); };

    // the state pass may be scheduled now: its CTAs take SMs as this grid's
    // CTAs leave them, and wait for this grid's completion before reading
    asm volatile("griddepcontrol.launch_dependents;");
    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_q, 1);
        mbar_init(bar_v, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_wout);
        prefetch_tmap(&tm_pout);
        prefetch_tmap(&tm_aqout);
        if ((int)blockIdx.x < pp.nitems) {
            issue_k(blockIdx.x, 0);
            issue_q(blockIdx.x);
            issue_v(blockIdx.x);
        }
    }
    if ((int)blockIdx.x < pp.nitems) load_gates(blockIdx.x);
    if (warp == 0) tmem_alloc(s_tmem, P_TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t ph_tma0 = 0, ph_tma1 = 0, ph_mma = 0, ph_q = 0, ph_v = 0;
    bool ok = true;

#define GDR_WAIT(bar, ph)                                                   \
    do {                                                                    \
        bool w_ok = mbar_wait(bar, ph);                                     \
        ph ^= 1u;                                                           \
        if (!__syncthreads_and(w_ok)) { ok = false; goto finish; }          \
    } while (0)

    for (int item = blockIdx.x, it = 0; item < pp.nitems; item += gridDim.x, ++it) {
        const int buf = it & 1;
        int ci, h, bb;
        coords(item, ci, h, bb);
        const int t0 = ci * C;
        const int n = min(C, T - t0);
        const uint32_t kb = sbase + P_OFF_K + buf * 16384u;
        const uint32_t vb = sbase + P_OFF_V;
        GDR_TRACE_P(0);
        // this item's gates (prefetched into registers) -> shared memory
        if (tid < C) {
            const bool valid = tid < n;
            s_alpha[tid] = valid ? bits_to_f32(g_a) : 1.f;
            s_beta[tid] = valid ? bits_to_f32(g_b) : 0.f;
        }
        // the next item's K: its buffer was last read by this CTA's previous P2
        const int next = item + gridDim.x;
        if (tid == 0 && next < pp.nitems) issue_k(next, buf ^ 1);
        if (next < pp.nitems) load_gates(next);
        __syncthreads();

        // decay scan: one warp, two tokens per lane
        if (warp == 0) {
            const int lane = tid;
            const float la0 = lg2_approx(s_alpha[2 * lane]);
            const float la1 = lg2_approx(s_alpha[2 * lane + 1]);
            float x = la0 + la1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            const float l1 = x, l0v = x - la1;
            s_l[2 * lane] = l0v;
            s_l[2 * lane + 1] = l1;
            s_g[2 * lane] = ex2_approx(l0v);
            s_g[2 * lane + 1] = ex2_approx(l1);
        }
        if (buf == 0) GDR_WAIT(&bar_tma[0], ph_tma0);  // also publishes the scan
        else GDR_WAIT(&bar_tma[1], ph_tma1);
        GDR_WAIT(bar_q, ph_q);
        GDR_TRACE_P(1);

        // ---- D1 = K K^T (lanes 0..63), Q K^T (lanes 64..127, columns 64..127) ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t koff = (ks >> 2) * 8192u + (ks & 3) * 32u;
                mma_bf16(tmem + P_TM_D1, sdesc_sw128(kb + koff, 16, 1024), sdesc_sw128(kb + koff, 16, 1024),
                         id, ks > 0);
                mma_bf16(tmem + P_TM_DQ, sdesc_sw128(sbase + P_OFF_Q - 8192 + koff, 16, 1024),
                         sdesc_sw128(kb + koff, 16, 1024), id, ks > 0);
            }
            mma_commit(bar_mma);
            // the previous item's stores must have left the staging tiles (A32, T32)
            bulk_wait_group_read0();
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        GDR_TRACE_P(2);

        // ---- A (fp32, strict lower) and its transposed 16 x 16 diagonal blocks ----
        if ((warp & 3) < 2) {
            const int r = row;  // 0..63
            float d[32];
            tmem_ld32(tmem + lane_base + P_TM_D1 + wg * 32, d);
            // A_rj = beta_r (k_r . k_j) 2^(l_r - l_j), j < r: every ratio at most 1
            const float rf = s_beta[r], lr = s_l[r];
            float* A32 = reinterpret_cast<float*>(sm + P_OFF_A32);
#pragma unroll
            for (int j4 = 0; j4 < 32; j4 += 4) {
                const int j = wg * 32 + j4;
                const float4 l4 = *reinterpret_cast<const float4*>(s_l + j);
                float4 x;
                x.x = j < r ? rf * ex2_approx(fminf(lr - l4.x, 0.f)) * d[j4] : 0.f;
                x.y = j + 1 < r ? rf * ex2_approx(fminf(lr - l4.y, 0.f)) * d[j4 + 1] : 0.f;
                x.z = j + 2 < r ? rf * ex2_approx(fminf(lr - l4.z, 0.f)) * d[j4 + 2] : 0.f;
                x.w = j + 3 < r ? rf * ex2_approx(fminf(lr - l4.w, 0.f)) * d[j4 + 3] : 0.f;
                d[j4] = x.x; d[j4 + 1] = x.y; d[j4 + 2] = x.z; d[j4 + 3] = x.w;
                *reinterpret_cast<float4*>(f32_at(A32, r, j)) = x;
            }
            const int I = r >> 4, rr = r & 15;
            if ((I >> 1) == wg) {
                float* at = reinterpret_cast<float*>(sm + P_OFF_SCR) + I * 272;
                if (I & 1) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) at[j * 16 + rr] = d[16 + j];
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) at[j * 16 + rr] = d[j];
                }
            }
        } else {
            // Aq_tj = (q_t . k_j) 2^(l_t - l_j), j <= t (bf16) -> staging over Q's first tile
            const int t = row - 64;
            float d[32];
            tmem_ld32(tmem + lane_base + P_TM_DQ + wg * 32, d);
            const float lt = s_l[t];
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                const int j0 = wg * 32 + c8 * 8;
                const float4 la = *reinterpret_cast<const float4*>(s_l + j0);
                const float4 lb = *reinterpret_cast<const float4*>(s_l + j0 + 4);
                const float lj[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    x[e] = j0 + e <= t ? d[c8 * 8 + e] * ex2_approx(fminf(lt - lj[e], 0.f)) : 0.f;
                st_chunk(sm + P_OFF_Q, sw128_chunk(t, wg * 4 + c8, 64), x);
            }
        }
        fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&tm_aqout, sm + P_OFF_Q, 0, h, t0, bb);
            bulk_commit_group();
        }
        GDR_TRACE_P(3);

        // ---- T = (I + A)^-1; L = T Diag(beta g), PRE = T Diag(beta) (bf16) ----------
        {
            float* A32 = reinterpret_cast<float*>(sm + P_OFF_A32);
            float* T32 = reinterpret_cast<float*>(sm + P_OFF_T32);
            solve_unit_lower(A32, T32, reinterpret_cast<float*>(sm + P_OFF_SCR), tid, warp);
            GDR_TRACE_P(4);
            const int r = tid & 63, q4 = tid >> 6;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c8 = q4 * 2 + cc;
                float x[8], y[8];
#pragma unroll
                for (int e4 = 0; e4 < 8; e4 += 4) {
                    const int j = c8 * 8 + e4;
                    // the block T[0:32, 32:64] is never written by the solve: it is zero
                    const float4 t4 = (j < 32 || r >= 32) ? *reinterpret_cast<const float4*>(f32_at(T32, r, j))
                                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float4 b4 = *reinterpret_cast<const float4*>(s_beta + j);
                    const float4 g4 = *reinterpret_cast<const float4*>(s_g + j);
                    y[e4] = t4.x * b4.x; y[e4 + 1] = t4.y * b4.y; y[e4 + 2] = t4.z * b4.z; y[e4 + 3] = t4.w * b4.w;
                    x[e4] = y[e4] * g4.x; x[e4 + 1] = y[e4 + 1] * g4.y; x[e4 + 2] = y[e4 + 2] * g4.z;
                    x[e4 + 3] = y[e4 + 3] * g4.w;
                }
                st_chunk(sm + P_OFF_A32, sw128_chunk(r, c8, 64), x);         // L
                st_chunk(sm + P_OFF_A32 + 8192, sw128_chunk(r, c8, 64), y);  // PRE
            }
        }
        fence_proxy_async();
        tc_fence_before();
        GDR_WAIT(bar_v, ph_v);  // V landed during the solve (also publishes L, PRE)

        // ---- D2 = L K (-> W), D3 = PRE V (-> P) ----------------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idW = idesc_bf16(128, 128, 0, 1);
            const uint32_t idP = idesc_bf16(128, dv, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                mma_bf16(tmem + P_TM_D2, sdesc_sw128(sbase + P_OFF_A32 + ks * 32u, 16, 1024),
                         sdesc_sw128(kb + ks * 2048u, 8192, 1024), idW, ks > 0);
                mma_bf16(tmem + P_TM_D3, sdesc_sw128(sbase + P_OFF_A32 + 8192 + ks * 32u, 16, 1024),
                         sdesc_sw128(vb + ks * 2048u, 8192, 1024), idP, ks > 0);
            }
            mma_commit(bar_mma);
        }
        GDR_TRACE_P(5);
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        if (tid == 0 && next < pp.nitems) {
            issue_v(next);            // the P product has read V
            bulk_wait_group_read0();  // the Aq store has left its staging tile over Q
            issue_q(next);
        }
        GDR_TRACE_P(6);

        // ---- -W and P -> staging tiles (rows 0..63; each warpgroup half the columns)
        if ((warp & 3) < 2) {
            const int r = row;
            float d[32], d1[32];
            tmem_ld32_async(tmem + lane_base + P_TM_D2 + wg * 64, d);
            tmem_ld32_async(tmem + lane_base + P_TM_D2 + wg * 64 + 32, d1);
            tmem_wait_ld();
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                float x[8];
                const float* dd = c8 < 4 ? d + c8 * 8 : d1 + (c8 - 4) * 8;
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = -dd[e];
                st_chunk(sm + P_OFF_A32, sw128_chunk(r, wg * 8 + c8, 64), x);
            }
            // P: each warpgroup dv / 2 columns (32 or 64)
            const int half = dv >> 1;
            tmem_ld32_async(tmem + lane_base + P_TM_D3 + wg * half, d);
            if (half == 64) tmem_ld32_async(tmem + lane_base + P_TM_D3 + wg * half + 32, d1);
            tmem_wait_ld();
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                if (c8 * 8 >= half) break;
                const float* dd = c8 < 4 ? d + c8 * 8 : d1 + (c8 - 4) * 8;
                st_chunk(sm + P_OFF_T32, sw128_chunk(r, (wg * half) / 8 + c8, 64), dd);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&tm_wout, sm + P_OFF_A32, 0, h, t0, bb);
            tma_store_4d(&tm_wout, sm + P_OFF_A32 + 8192, 64, h, t0, bb);
            for (int vt = 0; vt < nvt; ++vt) tma_store_4d(&tm_pout, sm + P_OFF_T32 + vt * 8192, vt * 64, h, t0, bb);
            bulk_commit_group();
        }
        GDR_TRACE_P(7);
    }

finish:
    if (!ok && tid == 0) flag_status(pp.d_status, GDR_DEVICE_TIMEOUT);
    if (tid == 0) bulk_wait_group0();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, P_TM_COLS);
#undef GDR_WAIT
}

// ---- pass 2 shared memory ---------------------------------------------------
// Inputs are triple-buffered (chunk ci + 2 loads while chunk ci runs); a stage
// holds [Q ; -W] (Q in rows 0..63, -W in rows 64..127, two 64-column blocks
// of 16 KB), K, this CTA's 64 columns of P and Aq (from the first pass; rows
// 0..63 of the Aq U operand, whose rows 64..127 are the next 8 KB, unused).
constexpr int S_NBUF = 3;
constexpr uint32_t S_STAGE = 65536;
constexpr uint32_t S_ST_QW = 0;         // [Q ; -W] bf16 [128 x 128]
constexpr uint32_t S_ST_K = 32768;      // K bf16 [64 x 128]
constexpr uint32_t S_ST_P = 49152;      // P slice bf16 [64 x 64]
constexpr uint32_t S_ST_AQ = 57344;     // Aq bf16 [64 x 64]
constexpr uint32_t S_OFF_SBF = S_NBUF * S_STAGE;     // S bf16 [128 x 64] (B operand, MN-major)
constexpr uint32_t S_OFF_U = S_OFF_SBF + 16384;      // U bf16 [64 x 64] (B operand of Aq U)
constexpr uint32_t S_OFF_U2 = S_OFF_U + 8192;        // Diag(g_{n-1}/g) U (B operand of K^T U)
constexpr uint32_t S_OFF_SMALL = S_OFF_U2 + 8192;
constexpr uint32_t S_SMEM_BYTES = S_OFF_SMALL + 2048 + 1024;
// TMEM columns: D3 [Q S ; -W S] and D5 (Aq U, lanes 0..63) alternate between
// two column sets by chunk parity, so chunk ci's outputs are written while
// chunk ci + 1 runs; D4 = K^T U'.
constexpr uint32_t S_TM_D3 = 0, S_TM_D4 = 192, S_TM_D5 = 256, S_TM_COLS = 512;
// Threads: warps 0..7 compute (thread t < 256: state row t & 127, columns
// 32 (t >> 7) .. + 31 of the CTA's 64); warp 8 issues every MMA and TMA load.
constexpr int S_NT = 288;
constexpr int S_BAR_CHUNK = 1;  // named barrier over the 256 compute threads

__device__ __forceinline__ bool named_bar_and(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Chunk step of the state pass. Only the two products that depend on the
// state are on the chain from one chunk to the next:
//   D3 = [Q ; -W] S             (U = P - W S, lanes 64..127, by warps 2, 3, 6, 7)
//   D4 = K^T Diag(g_{n-1}/g) U  (S <- g_{n-1} S + D4, all compute warps)
// The output's product follows D4:
//   D5 = [Aq ; .] U             (lanes 0..63: Aq U, Aq = masked (Q K^T) . 2^(l_r - l_j)
//                                formed by the first pass; with Q S it gives O of
//                                the chunk, written during the next chunk)
// Warp 8 issues them, each when its operands are in shared memory (mbarriers
// u_ready, s_ready), so no compute warp waits on MMA issue. D5 commits to one
// barrier per TMEM column set: a barrier completes every second chunk, so the
// warps that wait for one chunk's output can never see the next completion of
// the same barrier first.
// Optional checkpoints for the backward pass, written off the chunk chain:
// the state at every chunk start ([B, H, nchunks, 128, d_v]) and U = P - W S
// of every token ([B, T, H, d_v]; U = beta v - r, with r the token's erase
// read), both bf16: the backward reads them only as tensor-core operands and
// for one inner product per chunk.
struct Ckpt {
    __nv_bfloat16* ckS;
    __nv_bfloat16* up;
};

// CKPT: the backward pass's instantiation (checkpoints written, o not written);
// the forward's has none of that code.
template <bool CKPT>
__global__ void __launch_bounds__(S_NT, 1) state_gdn_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_p,
    const __grid_constant__ CUtensorMap tm_aq, const Params p, const Ckpt ck) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = (warp >> 2) & 1;
    const int row = tid & 127;             // TMEM lane / state row (compute threads)
    const bool lo = row < 64;              // warps 0, 1, 4, 5: lanes 0..63
    const int vt = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int hq = h / p.group;  // q / k head of this value head
    const int v0 = vt * NV;
    const int T = p.T, H = p.H;
    const int nchunks = (T + C - 1) / C;

    // per-chunk factors, three sets by chunk % 3 (written one chunk ahead,
    // read up to one chunk behind): g = 2^l (l the log2 prefix),
    // gcr = 2^(l_{n-1} - l), and g_{n-1}
    float* s_g3 = reinterpret_cast<float*>(sm + S_OFF_SMALL);   // [3][64]
    float* s_gcr3 = s_g3 + 192;                                  // [3][64]
    float* s_gC3 = s_g3 + 384;                                   // [3][4]
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + S_OFF_SMALL + 1600);  // [3]
    uint64_t* bar_w = bar_tma + 3;      // MMA commits
    uint64_t* bar_k = bar_tma + 4;
    uint64_t* bar_drain = bar_tma + 5;
    uint64_t* u_ready = bar_tma + 6;    // operands written (compute -> issuer)
    uint64_t* s_ready = bar_tma + 7;
    uint64_t* bar_a0 = bar_tma + 8;     // D5 commits, one per TMEM column set
    auto bar_a = [&](int set) { return bar_a0 + set; };
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + S_OFF_SMALL + 1696);
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bar_tma[i], 1);
        mbar_init(bar_w, 1);
        mbar_init(bar_k, 1);
        mbar_init(bar_a(0), 1);
        mbar_init(bar_a(1), 1);
        mbar_init(bar_drain, 1);
        mbar_init(u_ready, 128);
        mbar_init(s_ready, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_w);
        prefetch_tmap(&tm_p);
        prefetch_tmap(&tm_aq);
    }
    if (warp == 0) tmem_alloc(s_tmem, S_TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t sbase = smem_u32(sm);
    bool ok = true;

    constexpr int NH = NV / 2;
    float S[NH];
    if (warp < 8) {
        const float* s0 = p.S0 ? p.S0 + (((size_t)bb * H + h) * DK + row) * p.dv + v0 + wg * NH : nullptr;
#pragma unroll
        for (int j = 0; j < NH; j += 4) {
            float4 x = s0 ? *reinterpret_cast<const float4*>(s0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) st_chunk(sm + S_OFF_SBF, sw128_chunk(row, wg * 4 + ch, DK), &S[8 * ch]);
    }

    // decay scan of one chunk by warp 1 (two tokens per lane, alpha in
    // registers): factors set ci % 3
    auto bits_to_f32 = [](unsigned short u) { return __uint_as_float((uint32_t)u << 16); };
    unsigned short a_nx0 = 0x3F80, a_nx1 = 0x3F80;  // alpha of the next chunk to scan (bf16 1.0)
    auto load_alpha = [&](int ci) {
        const int t = ci * C + 2 * lane;
        const unsigned short* ap = (const unsigned short*)p.alpha;
        a_nx0 = t < T ? ap[((size_t)bb * T + t) * H + h] : (unsigned short)0x3F80;
        a_nx1 = t + 1 < T ? ap[((size_t)bb * T + t + 1) * H + h] : (unsigned short)0x3F80;
    };
    auto decay_scan = [&](int ci) {
        const int s3 = ci % 3;
        const float la0 = lg2_approx(bits_to_f32(a_nx0));
        const float la1 = lg2_approx(bits_to_f32(a_nx1));
        float x = la0 + la1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        const float l1 = x, l0v = x - la1;
        const float last = __shfl_sync(0xffffffffu, l1, 31);
        float* g = s_g3 + s3 * 64;
        float* gcr = s_gcr3 + s3 * 64;
        g[2 * lane] = ex2_approx(l0v);
        g[2 * lane + 1] = ex2_approx(l1);
        gcr[2 * lane] = ex2_approx(last - l0v);
        gcr[2 * lane + 1] = ex2_approx(last - l1);
        if (lane == 0) s_gC3[s3 * 4] = ex2_approx(last);
    };

    auto issue_loads = [&](int ci) {
        const int t0 = ci * C, buf = ci % S_NBUF;
        uint8_t* st = sm + buf * S_STAGE;
        mbar_expect_tx(&bar_tma[buf], 8u * 8192u);
        // [Q ; -W]: each 64-column block holds 128 rows (q rows 0..63, -W rows 64..127)
        tma_load_4d(st + S_ST_QW, &tm_q, &bar_tma[buf], 0, hq, t0, bb);
        tma_load_4d(st + S_ST_QW + 16384, &tm_q, &bar_tma[buf], 64, hq, t0, bb);
        tma_load_4d(st + S_ST_QW + 8192, &tm_w, &bar_tma[buf], 0, h, t0, bb);
        tma_load_4d(st + S_ST_QW + 16384 + 8192, &tm_w, &bar_tma[buf], 64, h, t0, bb);
        tma_load_4d(st + S_ST_K, &tm_k, &bar_tma[buf], 0, hq, t0, bb);
        tma_load_4d(st + S_ST_K + 8192, &tm_k, &bar_tma[buf], 64, hq, t0, bb);
        tma_load_4d(st + S_ST_P, &tm_p, &bar_tma[buf], v0, h, t0, bb);
        tma_load_4d(st + S_ST_AQ, &tm_aq, &bar_tma[buf], 0, h, t0, bb);
    };

    // the state's bf16 copy is read by the first MMA (async proxy)
    fence_proxy_async();
    tc_fence_before();
    // Everything above overlaps the first pass's tail (this grid may be
    // launched before that one completes: programmatic dependent launch);
    // the first pass's factors are read only after it has completed.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == 8 && lane == 0) {
        for (int ci = 0; ci < 2 && ci < nchunks; ++ci) issue_loads(ci);
    }
    if (warp == 1 && nchunks > 0) {
        load_alpha(0);
        decay_scan(0);
        if (nchunks > 1) load_alpha(1);
    }
    __syncthreads();

    int loads_issued = min(2, nchunks);  // issuer's bookkeeping
    if (warp == 8) {
        // ---------------- issuer warp: MMAs in chain order, TMA two chunks ahead --------
        bool iok = true;
        for (int ci = 0; ci < nchunks && iok; ++ci) {
            const int buf = ci % S_NBUF;
            const int par = ci & 1;
            const uint32_t ph = (uint32_t)(ci & 1);
            const uint32_t stb = sbase + buf * S_STAGE;
            const uint32_t qwb = stb + S_ST_QW, kb = stb + S_ST_K;
            // inputs landed, and (after the first chunk) the state copy is written
            iok = mbar_wait(&bar_tma[buf], (uint32_t)((ci / S_NBUF) & 1)) && iok;
            if (ci > 0) iok = mbar_wait(s_ready, (uint32_t)((ci - 1) & 1)) && iok;
            iok = __all_sync(0xffffffffu, iok);
            if (!iok) break;
            GDR_TRACE_S(0, 256);
            tc_fence_after();
            if (lane == 0) {
                const uint32_t idS = idesc_bf16(128, NV, 0, 1);
                const uint32_t d3 = S_TM_D3 + (uint32_t)par * 64u;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t koff = (ks >> 2) * 16384u + (ks & 3) * 32u;
                    mma_bf16(tmem + d3, sdesc_sw128(qwb + koff, 16, 1024),
                             sdesc_sw128(sbase + S_OFF_SBF + ks * 2048u, 8192, 1024), idS, ks > 0);
                }
                mma_commit(bar_w);
            }
            __syncwarp();
            // chunk ci + 2's inputs go to the stage of chunk ci - 1: its Aq tile's
            // reader (D5 of chunk ci - 1) has finished; every other reader of that
            // stage finished before the state copy of chunk ci was written
            if (ci > 0) {
                iok = __all_sync(0xffffffffu,
                                 mbar_wait(bar_a((ci - 1) & 1), (uint32_t)(((ci - 1) >> 1) & 1)) && iok);
                if (!iok) break;
            }
            if (lane == 0 && ci + 2 < nchunks) issue_loads(ci + 2);
            if (ci + 2 < nchunks) loads_issued = ci + 3;
            __syncwarp();
            // ---- D4 = K^T U', then D5 = [Aq ; .] U, once U is written --------------------
            iok = __all_sync(0xffffffffu, mbar_wait(u_ready, ph) && iok);
            if (!iok) break;
            GDR_TRACE_S(1, 256);
            tc_fence_after();
            if (lane == 0) {
                const uint32_t idM = idesc_bf16(128, NV, 1, 1);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + S_TM_D4, sdesc_sw128(kb + ks * 2048u, 8192, 1024),
                             sdesc_sw128(sbase + S_OFF_U2 + ks * 2048u, 8192, 1024), idM, ks > 0);
                mma_commit(bar_k);
                const uint32_t idA = idesc_bf16(128, NV, 0, 1);
                const uint32_t d5 = S_TM_D5 + (uint32_t)par * 64u;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + d5, sdesc_sw128(stb + S_ST_AQ + ks * 32u, 16, 1024),
                             sdesc_sw128(sbase + S_OFF_U + ks * 2048u, 8192, 1024), idA, ks > 0);
                mma_commit(bar_a(par));
            }
            __syncwarp();
        }
        if (!iok) {
            ok = false;
            if (lane == 0) {
                // before the block leaves (each wait bounded): the requested input
                // copies have landed and the issued MMAs have finished
                for (int ci = max(0, loads_issued - S_NBUF); ci < loads_issued; ++ci)
                    (void)mbar_wait(&bar_tma[ci % S_NBUF], (uint32_t)((ci / S_NBUF) & 1));
                mma_commit(bar_drain);
                (void)mbar_wait(bar_drain, 0);
            }
            __syncwarp();
        }
    } else {
        // ---------------- compute warps ----------------------------------------------
        bool w_ok = true;
        // O rows of chunk cj (lanes 0..63 of D3 and D5 in the column set of cj) -> global
        auto store_o = [&](int cj) {
            const int pj = cj & 1;
            const int t = cj * C + row;
            float d[32], d5[32];
            tmem_ld32_async(tmem + lane_base + S_TM_D3 + pj * 64 + wg * 32, d);
            tmem_ld32_async(tmem + lane_base + S_TM_D5 + pj * 64 + wg * 32, d5);
            tmem_wait_ld();
            if (t < T && !CKPT) {
                const float gr = s_g3[(cj % 3) * 64 + row];
                __nv_bfloat16* op = p.o + (((size_t)bb * T + t) * H + h) * p.dv + v0 + wg * 32;
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = fmaf(gr, d[c8 * 8 + e], d5[c8 * 8 + e]);
                    uint4 u;
                    u.x = pack_bf16x2(y[0], y[1]);
                    u.y = pack_bf16x2(y[2], y[3]);
                    u.z = pack_bf16x2(y[4], y[5]);
                    u.w = pack_bf16x2(y[6], y[7]);
                    *reinterpret_cast<uint4*>(op + c8 * 8) = u;
                }
            }
        };
        int ci = 0;
        for (; ci < nchunks; ++ci) {
            const int buf = ci % S_NBUF;
            const int par = ci & 1;
            const uint32_t ph = (uint32_t)(ci & 1);
            const int s3 = ci % 3;
            // the state at this chunk's start, for the backward pass (each thread
            // its row; the warps of lanes 64..127 once U has left)
            auto store_ck = [&]() {
                __nv_bfloat16* dst = ck.ckS + ((((size_t)bb * H + h) * nchunks + ci) * DK + row) * p.dv + v0 + wg * NH;
#pragma unroll
                for (int jj = 0; jj < NH; jj += 8)
                    *reinterpret_cast<uint4*>(dst + jj) =
                        make_uint4(pack_bf16x2(S[jj], S[jj + 1]), pack_bf16x2(S[jj + 2], S[jj + 3]),
                                   pack_bf16x2(S[jj + 4], S[jj + 5]), pack_bf16x2(S[jj + 6], S[jj + 7]));
            };
            if (CKPT && lo) store_ck();
            if (lo) {
                // ---- O of the previous chunk, the next decay scan ---------------------------
                if (ci > 0) {
                    w_ok = mbar_wait(bar_a((ci - 1) & 1), (uint32_t)(((ci - 1) >> 1) & 1)) && w_ok;
                    tc_fence_after();
                    store_o(ci - 1);
                }
                if (warp == 1 && ci + 1 < nchunks) {
                    decay_scan(ci + 1);
                    if (ci + 2 < nchunks) load_alpha(ci + 2);
                }
                GDR_TRACE_S(4, 0);
            } else {
                // ---- U = P - W S (lanes 64..127 of D3) -> U and U' -------------------------
                w_ok = mbar_wait(&bar_tma[buf], (uint32_t)((ci / S_NBUF) & 1)) && w_ok;  // P landed
                w_ok = mbar_wait(bar_w, ph) && w_ok;
                tc_fence_after();
                GDR_TRACE_S(7, 64);
                const int j = row - 64;  // token
                float d[32];
                tmem_ld32(tmem + lane_base + S_TM_D3 + (uint32_t)par * 64u + wg * 32, d);
                const float f = s_gcr3[s3 * 64 + j];
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    float x[8];
                    const uint32_t off = sw128_chunk(j, wg * 4 + c8, 64);
                    ld_chunk(sm + buf * S_STAGE + S_ST_P, off, x);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        x[e] += d[c8 * 8 + e];
                        if (CKPT) d[c8 * 8 + e] = x[e];  // U, kept for the checkpoint below
                    }
                    st_chunk(sm + S_OFF_U, off, x);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] *= f;
                    st_chunk(sm + S_OFF_U2, off, x);
                }
                fence_proxy_async();
                tc_fence_before();
                mbar_arrive(u_ready);
                if (CKPT) {  // U of every token and the chunk's start state, off the chain
                    if (ci * C + j < T) {
                        __nv_bfloat16* up = ck.up + (((size_t)bb * T + ci * C + j) * H + h) * p.dv + v0 + wg * 32;
#pragma unroll
                        for (int c8 = 0; c8 < 32; c8 += 8)
                            *reinterpret_cast<uint4*>(up + c8) =
                                make_uint4(pack_bf16x2(d[c8], d[c8 + 1]), pack_bf16x2(d[c8 + 2], d[c8 + 3]),
                                           pack_bf16x2(d[c8 + 4], d[c8 + 5]), pack_bf16x2(d[c8 + 6], d[c8 + 7]));
                    }
                    store_ck();
                }
            }
            // ---- S = g_{n-1} S + D4 (every compute warp: its lanes, half the columns) ----
            w_ok = mbar_wait(bar_k, ph) && w_ok;
            tc_fence_after();
            GDR_TRACE_S(5, 0);
            {
                float dS[32];
                tmem_ld32(tmem + lane_base + S_TM_D4 + wg * 32, dS);
                const float gC = s_gC3[s3 * 4];
#pragma unroll
                for (int jj = 0; jj < NH; ++jj) S[jj] = fmaf(gC, S[jj], dS[jj]);
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) st_chunk(sm + S_OFF_SBF, sw128_chunk(row, wg * 4 + ch, DK), &S[8 * ch]);
            }
            fence_proxy_async();  // the state copy feeds the next chunk's MMAs
            tc_fence_before();
            if (!named_bar_and(S_BAR_CHUNK, 256, w_ok)) break;
            GDR_TRACE_S(6, 0);
            if (tid == 0) mbar_arrive(s_ready);
        }
        if (ci < nchunks) ok = false;  // a wait gave up
        if (ok && lo && nchunks > 0) {
            ok = mbar_wait(bar_a((nchunks - 1) & 1), (uint32_t)(((nchunks - 1) >> 1) & 1));
            tc_fence_after();
            if (ok) store_o(nchunks - 1);
        }
        if (!named_bar_and(S_BAR_CHUNK, 256, ok)) ok = false;
        if (ok && p.ST) {
            float* st = p.ST + (((size_t)bb * H + h) * DK + row) * p.dv + v0 + wg * NH;
#pragma unroll
            for (int jj = 0; jj < NH; jj += 4)
                *reinterpret_cast<float4*>(st + jj) = make_float4(S[jj], S[jj + 1], S[jj + 2], S[jj + 3]);
        }
    }
    if (!ok && (tid == 0 || tid == 256)) flag_status(p.d_status, GDR_DEVICE_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, S_TM_COLS);
}

}  // namespace twopass

size_t twopass_workspace_bytes(int B, int T, int H, int dv) {
    return (size_t)B * T * H * (chunkc::DK + dv + chunkc::C) * sizeof(__nv_bfloat16);
}

// maps: q, k, v, then the workspace maps -W ([B,T,H,128]), P ([B,T,H,d_v]) and
// Aq ([B,T,H,64], the chunk's masked, decay-scaled Q K^T block row of each token).
// ckS, up: the backward pass's bf16 checkpoints (struct Ckpt; both or neither),
// or NULL: with them, o is not written.
cudaError_t launch_chunk_twopass_gdn(const CUtensorMap* maps, const CUtensorMap* ws_maps, void* ws,
                                     const void* alpha, const void* beta, const float* S0, void* o,
                                     float* ST, int* d_status, int B, int T, int H, int dv, int group,
                                     cudaStream_t st, __nv_bfloat16* ckS, __nv_bfloat16* up) {
    using namespace twopass;
    PrepParams pp;
    pp.alpha = alpha; pp.beta = beta;
    pp.d_status = d_status;
    pp.T = T; pp.H = H; pp.dv = dv;
    pp.group = group;
    const int nchunks = (T + C - 1) / C;
    pp.nitems = nchunks * H * B;
    cudaError_t e = cudaFuncSetAttribute(prep_gdn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int grid = min(pp.nitems, 2 * nsm);  // two resident CTAs per SM
    prep_gdn_kernel<<<grid, NT, P_SMEM_BYTES, st>>>(maps[0], maps[1], maps[2], ws_maps[0], ws_maps[1],
                                                    ws_maps[2], pp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    Params p;
    p.alpha = alpha; p.bg = beta; p.wg = nullptr;
    p.S0 = S0; p.o = (__nv_bfloat16*)o; p.ST = ST; p.d_status = d_status;
    p.B = B; p.T = T; p.H = H; p.dv = dv;
    p.akind = GDR_GATE_SCALAR; p.bkind = GDR_GATE_SCALAR; p.wkind = GDR_GATE_TIED;
    p.group = group;
    const bool ckpt = ckS != nullptr;
    e = ckpt ? cudaFuncSetAttribute(state_gdn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, S_SMEM_BYTES)
             : cudaFuncSetAttribute(state_gdn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, S_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(dv / NV, H, B);
    cfg.blockDim = dim3(S_NT, 1, 1);
    cfg.dynamicSmemBytes = S_SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap the prep tail
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    Ckpt ck;
    ck.ckS = ckS;
    ck.up = up;
    return ckpt ? cudaLaunchKernelEx(&cfg, state_gdn_kernel<true>, maps[0], maps[1], ws_maps[0], ws_maps[1],
                                     ws_maps[2], p, ck)
                : cudaLaunchKernelEx(&cfg, state_gdn_kernel<false>, maps[0], maps[1], ws_maps[0], ws_maps[1],
                                     ws_maps[2], p, ck);
}

}  // namespace gdr

#ifdef GDR_TRACE_PHASES
extern "C" int gdr_trace_twopass_read(unsigned long long* host, int n) {
    return (int)cudaMemcpyFromSymbol(host, gdr::twopass::g_trace2, sizeof(unsigned long long) * n);
}
#endif
