// Two-pass chunkwise forward for the Gated DeltaNet form (scalar decay per
// token, tied scalar b = w = beta) at key width d_k = 256 ("How Linear
// Attention Remembers", Table 1: Gated DeltaNet heads of d_k = d_v = 256), on
// sm_100a tensor cores.
//
// The chunk algebra is that of the d_k = 128 pair ("Erase-then-Delta
// Attention" abstract: chunkwise WY form with the decay absorbed into the
// erase factors; "Recurrent Memory: Write, Erase, Decay, Read" section 03 for
// the chunk reassociation):
//
//   pass 1 (persistent CTAs over all (chunk, head, batch) items, one per SM):
//     A  = Diag(beta) ((K K^T) . G) strict lower,  G_rj = g_r / g_j
//     T  = (I + A)^-1
//     -W = -T Diag(beta g) K                     -> workspace [B,T,H,256]
//     P  =  T Diag(beta) V                       -> workspace [B,T,H,d_v]
//     Aq = (Q K^T) . G, lower incl. the diagonal -> workspace [B,T,H,64]
//     K~ = Diag(g_{n-1} / g) K                   -> workspace [B,T,H,256]
//   pass 2 (one CTA per (batch, head, 64 columns of d_v), chunks in order):
//     U  = P - W S,  O = Diag(g) (Q S) + Aq U,  S' = g_{n-1} S + K~^T U
//
// What changes with d_k = 256: every K, Q, W tile is twice as wide (32 KB),
// the products over d_k take 16 K-steps, the state slice is 256 x 64 (two
// TMEM accumulators of 128 rows for K~^T U), and the shared memory no longer
// holds three input stages. Pass 1 therefore also writes K~ (so pass 2 keeps a
// single U tile for both of its U products) and pass 2 double-buffers its
// chain inputs ([Q ; -W], P) and single-buffers K~ and Aq, each reloaded as
// soon as its product has read it.
#include "chunk_common.cuh"

namespace gdr {
namespace twopass256 {

using namespace chunkc;

constexpr int DKW = 256;  // key width of this pair

// ---- pass 1 shared memory (bytes from a 1024-aligned base) ----------------
// M = 128 MMAs read A rows 64..127 beyond each 64-row operand; those rows land
// in the next region (garbage rows whose outputs are never read).
constexpr uint32_t P_OFF_K = 0;         // K [64 x 256] bf16, four 8 KB column blocks; 2 buffers
constexpr uint32_t P_OFF_Q = 65536;     // Q [64 x 256] bf16; its first block then stages Aq
constexpr uint32_t P_OFF_V = 98304;     // V [64 x d_v] bf16 (d_v <= 256)
constexpr uint32_t P_OFF_A32 = 131072;  // A fp32 [64 x 64]; then L, PRE bf16; with T32: -W staging
constexpr uint32_t P_OFF_T32 = 147456;  // T fp32 [64 x 64]
constexpr uint32_t P_OFF_PST = 163840;  // P staging [64 x d_v] bf16
constexpr uint32_t P_OFF_SCR = 196608;  // solve scratch fp32 (5 KB)
constexpr uint32_t P_OFF_SMALL = 201728;
constexpr uint32_t P_SMEM_BYTES = P_OFF_SMALL + 2048 + 1024;
// TMEM: D1 = K K^T (columns 0..63, lanes 0..63) and Q K^T (columns 64..127,
// lanes 64..127); then P (columns 0 .. d_v - 1) and -W (columns 256..511).
constexpr uint32_t P_TM_D1 = 0, P_TM_DQ = 64, P_TM_P = 0, P_TM_W = 256, P_TM_COLS = 512;

struct PrepParams {
    const void* alpha;
    const void* beta;
    int* d_status;
    int T, H, dv, nitems;
    int group;  // value heads per q/k head (q, k read at head h / group)
};

__global__ void __launch_bounds__(NT, 1) prep_gdn256_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                            const __grid_constant__ CUtensorMap tm_k,
                                                            const __grid_constant__ CUtensorMap tm_v,
                                                            const __grid_constant__ CUtensorMap tm_wout,
                                                            const __grid_constant__ CUtensorMap tm_pout,
                                                            const __grid_constant__ CUtensorMap tm_aqout,
                                                            const __grid_constant__ CUtensorMap tm_ktout,
                                                            const PrepParams pp) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, wg = warp >> 2, row = tid & 127;
    const int T = pp.T, H = pp.H, dv = pp.dv;
    const int nchunks = (T + C - 1) / C;
    const int nvt = dv / 64;

    float* s_beta = reinterpret_cast<float*>(sm + P_OFF_SMALL);
    float* s_alpha = s_beta + 64;
    float* s_l = s_beta + 128;    // log2 prefix of alpha over the chunk
    float* s_g = s_beta + 192;    // 2^l
    float* s_gcr = s_beta + 256;  // 2^(l_{n-1} - l)
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
        mbar_expect_tx(&bar_tma[buf], 4u * 8192u);
        for (int j = 0; j < 4; ++j)
            tma_load_4d(sm + P_OFF_K + buf * 32768 + j * 8192, &tm_k, &bar_tma[buf], j * 64, hq, ci * C, bb);
    };
    auto issue_q = [&](int item) {
        int ci, h, bb;
        coords(item, ci, h, bb);
        const int hq = h / pp.group;
        mbar_expect_tx(bar_q, 4u * 8192u);
        for (int j = 0; j < 4; ++j) tma_load_4d(sm + P_OFF_Q + j * 8192, &tm_q, bar_q, j * 64, hq, ci * C, bb);
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

    // the state pass may be scheduled now; it waits for this grid's completion
    // before its first workspace read
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
        prefetch_tmap(&tm_ktout);
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
        const uint32_t kb = sbase + P_OFF_K + buf * 32768u;
        const uint32_t vb = sbase + P_OFF_V;
        if (tid < C) {
            const bool valid = tid < n;
            s_alpha[tid] = valid ? bits_to_f32(g_a) : 1.f;
            s_beta[tid] = valid ? bits_to_f32(g_b) : 0.f;
        }
        const int next = item + gridDim.x;
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
            const float last = __shfl_sync(0xffffffffu, l1, 31);
            s_l[2 * lane] = l0v;
            s_l[2 * lane + 1] = l1;
            s_g[2 * lane] = ex2_approx(l0v);
            s_g[2 * lane + 1] = ex2_approx(l1);
            s_gcr[2 * lane] = ex2_approx(last - l0v);
            s_gcr[2 * lane + 1] = ex2_approx(last - l1);
        }
        if (buf == 0) GDR_WAIT(&bar_tma[0], ph_tma0);  // also publishes the scan
        else GDR_WAIT(&bar_tma[1], ph_tma1);
        GDR_WAIT(bar_q, ph_q);

        // ---- D1 = K K^T (lanes 0..63), Q K^T (lanes 64..127, columns 64..127) ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 16; ++ks) {
                const uint32_t koff = (ks >> 2) * 8192u + (ks & 3) * 32u;
                mma_bf16(tmem + P_TM_D1, sdesc_sw128(kb + koff, 16, 1024), sdesc_sw128(kb + koff, 16, 1024),
                         id, ks > 0);
                mma_bf16(tmem + P_TM_DQ, sdesc_sw128(sbase + P_OFF_Q - 8192 + koff, 16, 1024),
                         sdesc_sw128(kb + koff, 16, 1024), id, ks > 0);
            }
            mma_commit(bar_mma);
            // the previous item's stores (-W and K~ out of the A32 / T32 tiles and
            // the other K buffer, P out of its staging tile) have read shared memory:
            // the next item's K may load into that buffer
            bulk_wait_group_read0();
            if (next < pp.nitems) issue_k(next, buf ^ 1);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();

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
            // Aq_tj = (q_t . k_j) 2^(l_t - l_j), j <= t (bf16) -> staging over Q's first block
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

        // ---- T = (I + A)^-1; L = T Diag(beta g), PRE = T Diag(beta) (bf16) ----------
        {
            float* A32 = reinterpret_cast<float*>(sm + P_OFF_A32);
            float* T32 = reinterpret_cast<float*>(sm + P_OFF_T32);
            solve_unit_lower(A32, T32, reinterpret_cast<float*>(sm + P_OFF_SCR), tid, warp);
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

        // ---- -W (N = 256) = L K, P (N = d_v) = PRE V ---------------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idW = idesc_bf16(128, DKW, 0, 1);
            const uint32_t idP = idesc_bf16(128, dv, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                mma_bf16(tmem + P_TM_W, sdesc_sw128(sbase + P_OFF_A32 + ks * 32u, 16, 1024),
                         sdesc_sw128(kb + ks * 2048u, 8192, 1024), idW, ks > 0);
                mma_bf16(tmem + P_TM_P, sdesc_sw128(sbase + P_OFF_A32 + 8192 + ks * 32u, 16, 1024),
                         sdesc_sw128(vb + ks * 2048u, 8192, 1024), idP, ks > 0);
            }
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        if (tid == 0 && next < pp.nitems) {
            issue_v(next);            // the P product has read V
            bulk_wait_group_read0();  // the Aq store has left its staging tile over Q
            issue_q(next);
        }

        if ((warp & 3) < 2) {
            // ---- -W -> staging over A32 / T32, P -> its staging tile (rows 0..63) ----
            const int r = row;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float d[32], d1[32];
                const uint32_t c0 = (uint32_t)(wg * 128 + hh * 64);
                tmem_ld32_async(tmem + lane_base + P_TM_W + c0, d);
                tmem_ld32_async(tmem + lane_base + P_TM_W + c0 + 32, d1);
                tmem_wait_ld();
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    float x[8];
                    const float* dd = c8 < 4 ? d + c8 * 8 : d1 + (c8 - 4) * 8;
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = -dd[e];
                    st_chunk(sm + P_OFF_A32, sw128_chunk(r, (int)(c0 >> 3) + c8, 64), x);
                }
            }
            // P: each warpgroup d_v / 2 columns, 32 at a time
            const int half = dv >> 1;
            for (int c0 = 0; c0 < half; c0 += 32) {
                float d[32];
                tmem_ld32(tmem + lane_base + P_TM_P + wg * half + c0, d);
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8)
                    st_chunk(sm + P_OFF_PST, sw128_chunk(r, (wg * half + c0) / 8 + c8, 64), d + c8 * 8);
            }
        } else {
            // ---- K~ = Diag(g_{n-1} / g) K in place (the MMAs have read K) ---------------
            // 2048 16-byte pieces of four 64 x 64 blocks; a piece's row is its
            // 128-byte line within the block (the swizzle permutes pieces within
            // a line), so each piece is scaled by its token's factor.
            uint8_t* kt = sm + P_OFF_K + buf * 32768;
            const int uu = wg ? tid - 128 : tid - 64;  // 0..127 over warps 2, 3, 6, 7
#pragma unroll 4
            for (int i = 0; i < 16; ++i) {
                const uint32_t off = (uint32_t)(uu + 128 * i) * 16u;
                const float f = s_gcr[(off & 8191u) >> 7];
                float x[8];
                ld_chunk(kt, off, x);
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] *= f;
                st_chunk(kt, off, x);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            for (int j = 0; j < 4; ++j) tma_store_4d(&tm_wout, sm + P_OFF_A32 + j * 8192, j * 64, h, t0, bb);
            for (int vt = 0; vt < nvt; ++vt) tma_store_4d(&tm_pout, sm + P_OFF_PST + vt * 8192, vt * 64, h, t0, bb);
            for (int j = 0; j < 4; ++j)
                tma_store_4d(&tm_ktout, sm + P_OFF_K + buf * 32768 + j * 8192, j * 64, h, t0, bb);
            bulk_commit_group();
        }
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
// Two stages of the chain inputs: [Q ; -W] (per 64-column block j of d_k, Q at
// 16 KB j and -W at 16 KB j + 8 KB, so one M = 128 operand holds both) and
// this CTA's 64 columns of P. K~ and Aq have one buffer each. Aq's garbage rows
// (the A operand is 128 rows) are the next 8 KB, the state copy.
constexpr uint32_t S_STAGE = 73728;
constexpr uint32_t S_ST_QW = 0;                       // [Q ; -W] bf16, four 16 KB blocks
constexpr uint32_t S_ST_P = 65536;                    // P slice bf16 [64 x 64]
constexpr uint32_t S_OFF_KT = 2 * S_STAGE;            // K~ bf16 [64 x 256]
constexpr uint32_t S_OFF_AQ = S_OFF_KT + 32768;       // Aq bf16 [64 x 64]
constexpr uint32_t S_OFF_SBF = S_OFF_AQ + 8192;       // S bf16 [256 x 64] (B operand, MN-major)
constexpr uint32_t S_OFF_U = S_OFF_SBF + 32768;       // U bf16 [64 x 64] (B operand of both U products)
constexpr uint32_t S_OFF_SMALL = S_OFF_U + 8192;
constexpr uint32_t S_SMEM_BYTES = S_OFF_SMALL + 1024 + 1024;
// TMEM: D3 = [Q S ; -W S] and D5 = Aq U in two column sets by chunk parity;
// D4 = K~^T U as two 128-row accumulators (state rows 0..127, 128..255).
constexpr uint32_t S_TM_D3 = 0, S_TM_D4 = 128, S_TM_D5 = 256, S_TM_COLS = 512;
constexpr int S_NT = 288;        // warps 0..7 compute, warp 8 issues every MMA and TMA load
constexpr int S_BAR_CHUNK = 1;   // named barrier over the 256 compute threads

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

// Chunk step (as in the d_k = 128 state pass): D3 = [Q ; -W] S (16 MMAs over
// d_k), U = P - W S by the warps of lanes 64..127, D4 = K~^T U (two 128-row
// halves), S <- g_{n-1} S + D4 by every compute warp (thread: state rows r and
// r + 128, 32 columns), D5 = Aq U for the output, written during the next
// chunk. D5 commits to one barrier per TMEM column set (a barrier completes
// every second chunk, so a wait can never see the next completion first).
__global__ void __launch_bounds__(S_NT, 1) state_gdn256_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_w,
    const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_aq,
    const __grid_constant__ CUtensorMap tm_kt, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = (warp >> 2) & 1;
    const int row = tid & 127;  // TMEM lane (compute threads)
    const bool lo = row < 64;   // warps 0, 1, 4, 5: lanes 0..63 (output rows)
    const int vt = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int hq = h / p.group;
    const int v0 = vt * NV;
    const int T = p.T, H = p.H;
    const int nchunks = (T + C - 1) / C;

    // per-chunk factors, three sets by chunk % 3 (written one chunk ahead, read
    // up to one chunk behind): g = 2^l and g_{n-1}
    float* s_g3 = reinterpret_cast<float*>(sm + S_OFF_SMALL);  // [3][64]
    float* s_gC3 = s_g3 + 192;                                  // [3][4]
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + S_OFF_SMALL + 832);  // [2] stages
    uint64_t* bar_kt = bar_tma + 2;   // K~ landed
    uint64_t* bar_aq = bar_tma + 3;   // Aq landed
    uint64_t* bar_w = bar_tma + 4;    // MMA commits
    uint64_t* bar_k = bar_tma + 5;
    uint64_t* bar_drain = bar_tma + 6;
    uint64_t* u_ready = bar_tma + 7;  // operands written (compute -> issuer)
    uint64_t* s_ready = bar_tma + 8;
    uint64_t* bar_a0 = bar_tma + 9;   // D5 commits, one per TMEM column set
    auto bar_a = [&](int set) { return bar_a0 + set; };
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + S_OFF_SMALL + 928);
    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(bar_kt, 1);
        mbar_init(bar_aq, 1);
        mbar_init(bar_w, 1);
        mbar_init(bar_k, 1);
        mbar_init(bar_drain, 1);
        mbar_init(u_ready, 128);
        mbar_init(s_ready, 1);
        mbar_init(bar_a(0), 1);
        mbar_init(bar_a(1), 1);
        fence_barrier_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_w);
        prefetch_tmap(&tm_p);
        prefetch_tmap(&tm_aq);
        prefetch_tmap(&tm_kt);
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
    float Slo[NH], Shi[NH];  // state rows `row` and `row + 128`, columns v0 + 32 wg ..
    if (warp < 8) {
        const float* s0 = p.S0 ? p.S0 + (((size_t)bb * H + h) * DKW + row) * p.dv + v0 + wg * NH : nullptr;
        const size_t hi = (size_t)128 * p.dv;
#pragma unroll
        for (int j = 0; j < NH; j += 4) {
            float4 x = s0 ? *reinterpret_cast<const float4*>(s0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            float4 y = s0 ? *reinterpret_cast<const float4*>(s0 + hi + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            Slo[j] = x.x; Slo[j + 1] = x.y; Slo[j + 2] = x.z; Slo[j + 3] = x.w;
            Shi[j] = y.x; Shi[j + 1] = y.y; Shi[j + 2] = y.z; Shi[j + 3] = y.w;
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            st_chunk(sm + S_OFF_SBF, sw128_chunk(row, wg * 4 + ch, DKW), &Slo[8 * ch]);
            st_chunk(sm + S_OFF_SBF, sw128_chunk(row + 128, wg * 4 + ch, DKW), &Shi[8 * ch]);
        }
    }

    // decay scan of one chunk by warp 1 (two tokens per lane): factors set ci % 3
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
        g[2 * lane] = ex2_approx(l0v);
        g[2 * lane + 1] = ex2_approx(l1);
        if (lane == 0) s_gC3[s3 * 4] = ex2_approx(last);
    };

    auto issue_stage = [&](int ci) {
        const int t0 = ci * C, buf = ci & 1;
        uint8_t* st = sm + buf * S_STAGE;
        mbar_expect_tx(&bar_tma[buf], 9u * 8192u);
        for (int j = 0; j < 4; ++j) {
            tma_load_4d(st + S_ST_QW + j * 16384, &tm_q, &bar_tma[buf], j * 64, hq, t0, bb);
            tma_load_4d(st + S_ST_QW + j * 16384 + 8192, &tm_w, &bar_tma[buf], j * 64, h, t0, bb);
        }
        tma_load_4d(st + S_ST_P, &tm_p, &bar_tma[buf], v0, h, t0, bb);
    };
    auto issue_kt = [&](int ci) {
        mbar_expect_tx(bar_kt, 4u * 8192u);
        for (int j = 0; j < 4; ++j) tma_load_4d(sm + S_OFF_KT + j * 8192, &tm_kt, bar_kt, j * 64, h, ci * C, bb);
    };
    auto issue_aq = [&](int ci) {
        mbar_expect_tx(bar_aq, 8192u);
        tma_load_4d(sm + S_OFF_AQ, &tm_aq, bar_aq, 0, h, ci * C, bb);
    };

    // the state's bf16 copy is read by the first MMA (async proxy)
    fence_proxy_async();
    tc_fence_before();
    // everything above overlaps the first pass's tail; its outputs are read
    // only after it has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == 8 && lane == 0 && nchunks > 0) {
        issue_stage(0);
        issue_kt(0);
        issue_aq(0);
    }
    if (warp == 1 && nchunks > 0) {
        load_alpha(0);
        decay_scan(0);
        if (nchunks > 1) load_alpha(1);
    }
    __syncthreads();

    if (warp == 8) {
        // ---------------- issuer warp --------------------------------------------------
        bool iok = true;
        // chunks whose loads were requested, per buffer kind (for the drain)
        int st_issued = nchunks > 0 ? 1 : 0, kt_issued = st_issued, aq_issued = st_issued;
        for (int ci = 0; ci < nchunks && iok; ++ci) {
            const int buf = ci & 1;
            const int par = ci & 1;
            const uint32_t ph = (uint32_t)(ci & 1);
            const uint32_t stb = sbase + buf * S_STAGE;
            iok = mbar_wait(&bar_tma[buf], (uint32_t)((ci >> 1) & 1)) && iok;
            if (ci > 0) iok = mbar_wait(s_ready, (uint32_t)((ci - 1) & 1)) && iok;
            iok = __all_sync(0xffffffffu, iok);
            if (!iok) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t idS = idesc_bf16(128, NV, 0, 1);
                const uint32_t d3 = S_TM_D3 + (uint32_t)par * 64u;
#pragma unroll
                for (int ks = 0; ks < 16; ++ks) {
                    const uint32_t koff = (ks >> 2) * 16384u + (ks & 3) * 32u;
                    mma_bf16(tmem + d3, sdesc_sw128(stb + S_ST_QW + koff, 16, 1024),
                             sdesc_sw128(sbase + S_OFF_SBF + ks * 2048u, 8192, 1024), idS, ks > 0);
                }
                mma_commit(bar_w);
                // the other stage was read by chunk ci - 1's D3 and U unload, both
                // finished before its state update (s_ready above)
                if (ci + 1 < nchunks) issue_stage(ci + 1);
            }
            if (ci + 1 < nchunks) st_issued = ci + 2;
            __syncwarp();
            // ---- D4 = K~^T U once U is written and K~ has landed, then D5 = Aq U ---------
            iok = __all_sync(0xffffffffu, mbar_wait(u_ready, ph) && mbar_wait(bar_kt, ph) && iok);
            if (!iok) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t idM = idesc_bf16(128, NV, 1, 1);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16(tmem + S_TM_D4 + hh * 64, sdesc_sw128(sbase + S_OFF_KT + hh * 16384u + ks * 2048u, 8192, 1024),
                                 sdesc_sw128(sbase + S_OFF_U + ks * 2048u, 8192, 1024), idM, ks > 0);
                mma_commit(bar_k);
            }
            __syncwarp();
            iok = __all_sync(0xffffffffu, mbar_wait(bar_aq, ph) && iok);
            if (!iok) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t idA = idesc_bf16(128, NV, 0, 1);
                const uint32_t d5 = S_TM_D5 + (uint32_t)par * 64u;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + d5, sdesc_sw128(sbase + S_OFF_AQ + ks * 32u, 16, 1024),
                             sdesc_sw128(sbase + S_OFF_U + ks * 2048u, 8192, 1024), idA, ks > 0);
                mma_commit(bar_a(par));
            }
            __syncwarp();
            if (ci + 1 < nchunks) {
                // the next K~ once D4 has read this one, the next Aq once D5 has
                iok = __all_sync(0xffffffffu, mbar_wait(bar_k, ph) && iok);
                if (!iok) break;
                if (lane == 0) issue_kt(ci + 1);
                kt_issued = ci + 2;
                iok = __all_sync(0xffffffffu, mbar_wait(bar_a(par), (uint32_t)((ci >> 1) & 1)) && iok);
                if (!iok) break;
                if (lane == 0) issue_aq(ci + 1);
                aq_issued = ci + 2;
                __syncwarp();
            }
        }
        if (!iok) {
            ok = false;
            if (lane == 0) {
                // before the block leaves (each wait bounded): the last requested copy
                // into every buffer has landed and the issued MMAs have finished
                for (int c = max(0, st_issued - 2); c < st_issued; ++c)
                    (void)mbar_wait(&bar_tma[c & 1], (uint32_t)((c >> 1) & 1));
                if (kt_issued > 0) (void)mbar_wait(bar_kt, (uint32_t)((kt_issued - 1) & 1));
                if (aq_issued > 0) (void)mbar_wait(bar_aq, (uint32_t)((aq_issued - 1) & 1));
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
            if (t < T) {
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
            const int buf = ci & 1;
            const int par = ci & 1;
            const uint32_t ph = (uint32_t)(ci & 1);
            const int s3 = ci % 3;
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
            } else {
                // ---- U = P - W S (lanes 64..127 of D3) ---------------------------------------
                w_ok = mbar_wait(&bar_tma[buf], (uint32_t)((ci >> 1) & 1)) && w_ok;  // P landed
                w_ok = mbar_wait(bar_w, ph) && w_ok;
                tc_fence_after();
                const int j = row - 64;  // token
                float d[32];
                tmem_ld32(tmem + lane_base + S_TM_D3 + (uint32_t)par * 64u + wg * 32, d);
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    float x[8];
                    const uint32_t off = sw128_chunk(j, wg * 4 + c8, 64);
                    ld_chunk(sm + buf * S_STAGE + S_ST_P, off, x);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] += d[c8 * 8 + e];
                    st_chunk(sm + S_OFF_U, off, x);
                }
                fence_proxy_async();
                tc_fence_before();
                mbar_arrive(u_ready);
            }
            // ---- S = g_{n-1} S + D4 (every compute warp: rows r, r + 128; 32 columns) ----
            w_ok = mbar_wait(bar_k, ph) && w_ok;
            tc_fence_after();
            {
                const float gC = s_gC3[s3 * 4];
                float dS[32];
                tmem_ld32(tmem + lane_base + S_TM_D4 + wg * 32, dS);
#pragma unroll
                for (int jj = 0; jj < NH; ++jj) Slo[jj] = fmaf(gC, Slo[jj], dS[jj]);
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) st_chunk(sm + S_OFF_SBF, sw128_chunk(row, wg * 4 + ch, DKW), &Slo[8 * ch]);
                tmem_ld32(tmem + lane_base + S_TM_D4 + 64 + wg * 32, dS);
#pragma unroll
                for (int jj = 0; jj < NH; ++jj) Shi[jj] = fmaf(gC, Shi[jj], dS[jj]);
#pragma unroll
                for (int ch = 0; ch < 4; ++ch)
                    st_chunk(sm + S_OFF_SBF, sw128_chunk(row + 128, wg * 4 + ch, DKW), &Shi[8 * ch]);
            }
            fence_proxy_async();  // the state copy feeds the next chunk's MMAs
            tc_fence_before();
            if (!named_bar_and(S_BAR_CHUNK, 256, w_ok)) break;
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
            float* st = p.ST + (((size_t)bb * H + h) * DKW + row) * p.dv + v0 + wg * NH;
            const size_t hi = (size_t)128 * p.dv;
#pragma unroll
            for (int jj = 0; jj < NH; jj += 4) {
                *reinterpret_cast<float4*>(st + jj) = make_float4(Slo[jj], Slo[jj + 1], Slo[jj + 2], Slo[jj + 3]);
                *reinterpret_cast<float4*>(st + hi + jj) = make_float4(Shi[jj], Shi[jj + 1], Shi[jj + 2], Shi[jj + 3]);
            }
        }
    }
    if (!ok && (tid == 0 || tid == 256)) flag_status(p.d_status, GDR_DEVICE_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, S_TM_COLS);
}

}  // namespace twopass256

// Workspace per token-head: -W (256), P (d_v), the chunk's Aq row (64), K~ (256), bf16.
size_t twopass256_workspace_bytes(int B, int T, int H, int dv) {
    return (size_t)B * T * H * (twopass256::DKW + dv + chunkc::C + twopass256::DKW) * sizeof(__nv_bfloat16);
}

// maps: q, k ([B,T,H/group,256]) and v ([B,T,H,d_v]); ws_maps: -W ([B,T,H,256]),
// P ([B,T,H,d_v]), Aq ([B,T,H,64]), K~ ([B,T,H,256]) in the workspace.
cudaError_t launch_chunk_twopass_gdn256(const CUtensorMap* maps, const CUtensorMap* ws_maps,
                                        const void* alpha, const void* beta, const float* S0, void* o,
                                        float* ST, int* d_status, int B, int T, int H, int dv, int group,
                                        cudaStream_t st) {
    using namespace twopass256;
    if (dv < 64 || dv > 256 || dv % 64 != 0) return cudaErrorInvalidValue;
    PrepParams pp;
    pp.alpha = alpha; pp.beta = beta;
    pp.d_status = d_status;
    pp.T = T; pp.H = H; pp.dv = dv;
    pp.group = group;
    const int nchunks = (T + C - 1) / C;
    pp.nitems = nchunks * H * B;
    cudaError_t e = cudaFuncSetAttribute(prep_gdn256_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int grid = min(pp.nitems, nsm);  // one resident CTA per SM (512 TMEM columns)
    prep_gdn256_kernel<<<grid, NT, P_SMEM_BYTES, st>>>(maps[0], maps[1], maps[2], ws_maps[0], ws_maps[1],
                                                       ws_maps[2], ws_maps[3], pp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    Params p;
    p.q = nullptr; p.k = nullptr; p.v = nullptr;
    p.alpha = alpha; p.bg = beta; p.wg = nullptr;
    p.S0 = S0; p.o = (__nv_bfloat16*)o; p.ST = ST; p.d_status = d_status;
    p.B = B; p.T = T; p.H = H; p.dv = dv;
    p.akind = GDR_GATE_SCALAR; p.bkind = GDR_GATE_SCALAR; p.wkind = GDR_GATE_TIED;
    p.group = group;
    e = cudaFuncSetAttribute(state_gdn256_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, S_SMEM_BYTES);
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
    return cudaLaunchKernelEx(&cfg, state_gdn256_kernel, maps[0], ws_maps[0], ws_maps[1], ws_maps[2],
                              ws_maps[3], p);
}

}  // namespace gdr
