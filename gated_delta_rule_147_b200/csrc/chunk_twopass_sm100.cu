// Two-pass chunkwise forward for the Gated DeltaNet form (scalar decay per
// token, tied scalar b = w = beta) on sm_100a tensor cores.
//
// The per-chunk WY/UT factors depend only on the chunk's own keys, values and
// gates, not on the state ("Erase-then-Delta Attention" abstract: chunkwise
// WY form with the decay absorbed into the erase factors; "Recurrent Memory:
// Write, Erase, Decay, Read" section 03 for the chunk reassociation). So the
// forward runs in two passes:
//
//   pass 1 (prep, one CTA per chunk, all chunks of all heads in parallel):
//     A  = Diag(beta rowf) (K K^T) Diag(colf)       strict lower
//     T  = (I + A)^-1
//     -W = -T Diag(beta g) K                        -> workspace [B,T,H,128] bf16
//     P  =  T Diag(beta) V                          -> workspace [B,T,H,d_v] bf16
//   pass 2 (state, one CTA per (batch, head, 64 columns of d_v), chunks in order):
//     U  = P - W S                                  (MMA [-W ; Q] S, plus P)
//     Aq = Diag(rowf) (Q K^T) Diag(colf)            lower   (same MMA batch)
//     O  = Diag(g) (Q S) + Aq U
//     S' = g_{n-1} S + (Diag(g_{n-1}/g) K)^T U
// with l_r the prefix sum of log2 alpha over the chunk, g_r = 2^l_r, and the
// bounded factors rowf_r = 2^(l_r - ref), colf_r = 2^(ref - l_r) around the
// chunk's reference ref = (l_0 + l_{n-1}) / 2.
//
// Pass 2's per-chunk chain is two MMA round trips; the triangular solve and
// the W / P products (most of the single-pass kernel's chain) run in pass 1
// with every chunk of every head in flight at once.
#include "chunk_common.cuh"

namespace gdr {
namespace twopass {

using namespace chunkc;

// ---- pass 1 shared memory (bytes from a 1024-aligned base) ----------------
// M = 128 MMAs read A rows 64..127 beyond each 64-row operand; those rows
// land in the next region (garbage rows whose outputs are never read).
constexpr uint32_t P_OFF_K = 0;        // K [64 x 128] bf16, two 8 KB column halves
constexpr uint32_t P_OFF_V = 16384;    // V [64 x d_v] bf16, d_v / 64 tiles of 8 KB (d_v <= 128)
constexpr uint32_t P_OFF_A32 = 32768;  // A fp32 [64 x 64]; after the solve L (8 KB) and PRE (8 KB)
constexpr uint32_t P_OFF_T32 = 49152;  // T fp32 [64 x 64]
constexpr uint32_t P_OFF_SCR = 65536;  // solve scratch fp32 (5 KB)
constexpr uint32_t P_OFF_SMALL = 70656;
constexpr uint32_t P_SMEM_BYTES = P_OFF_SMALL + 2048 + 1024;
constexpr uint32_t P_TM_D1 = 0, P_TM_D3 = 0, P_TM_D2 = 128, P_TM_COLS = 256;

struct PrepParams {
    const void* alpha;
    const void* beta;
    __nv_bfloat16* wneg;  // [B, T, H, 128]
    __nv_bfloat16* p;     // [B, T, H, d_v]
    int* d_status;
    int T, H, dv;
};

__global__ void __launch_bounds__(NT, 2) prep_gdn_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                         const __grid_constant__ CUtensorMap tm_v,
                                                         const PrepParams pp) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, wg = warp >> 2, row = tid & 127;
    const int ci = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int T = pp.T, H = pp.H, dv = pp.dv;
    const int t0 = ci * C;
    const int n = min(C, T - t0);
    const int nvt = dv / 64;

    float* s_beta = reinterpret_cast<float*>(sm + P_OFF_SMALL);
    float* s_rowf = s_beta + 64;
    float* s_colf = s_beta + 128;
    float* s_g = s_beta + 192;
    float* s_alpha = s_beta + 256;
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + P_OFF_SMALL + 1280);
    uint64_t* bar_mma = bar_tma + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + P_OFF_SMALL + 1296);
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
        mbar_expect_tx(bar_tma, (uint32_t)(2 + nvt) * 8192u);
        tma_load_4d(sm + P_OFF_K, &tm_k, bar_tma, 0, h, t0, bb);
        tma_load_4d(sm + P_OFF_K + 8192, &tm_k, bar_tma, 64, h, t0, bb);
        for (int vt = 0; vt < nvt; ++vt)
            tma_load_4d(sm + P_OFF_V + vt * 8192, &tm_v, bar_tma, vt * 64, h, t0, bb);
    }
    if (warp == 0) tmem_alloc(s_tmem, P_TM_COLS);
    if (tid < C) {
        const bool valid = tid < n;
        const size_t gi = ((size_t)bb * T + (valid ? t0 + tid : t0)) * H + h;
        const float a = to_f32(reinterpret_cast<const __nv_bfloat16*>(pp.alpha)[gi]);
        const float be = to_f32(reinterpret_cast<const __nv_bfloat16*>(pp.beta)[gi]);
        s_alpha[tid] = valid ? a : 1.f;
        s_beta[tid] = valid ? be : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t ph_tma = 0, ph_mma = 0;
    bool ok = true;

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
        const float first = __shfl_sync(0xffffffffu, l0v, 0);
        const float last = __shfl_sync(0xffffffffu, l1, 31);
        const float ref = 0.5f * (first + last);
        s_rowf[2 * lane] = ex2_approx(l0v - ref);
        s_rowf[2 * lane + 1] = ex2_approx(l1 - ref);
        s_colf[2 * lane] = ex2_approx(ref - l0v);
        s_colf[2 * lane + 1] = ex2_approx(ref - l1);
        s_g[2 * lane] = ex2_approx(l0v);
        s_g[2 * lane + 1] = ex2_approx(l1);
        if (lane == 0 && first - last > 230.f) flag_status(pp.d_status, GDR_DEVICE_DECAY_RANGE);
    }

#define GDR_WAIT(bar, ph)                                                   \
    do {                                                                    \
        bool w_ok = mbar_wait(bar, ph);                                     \
        ph ^= 1u;                                                           \
        if (!__syncthreads_and(w_ok)) { ok = false; goto finish; }          \
    } while (0)

    GDR_WAIT(bar_tma, ph_tma);  // also publishes the scan

    // ---- D1 = K K^T ---------------------------------------------------------
    if (tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t koff = (ks >> 2) * 8192u + (ks & 3) * 32u;
            mma_bf16(tmem + P_TM_D1, sdesc_sw128(sbase + P_OFF_K + koff, 16, 1024),
                     sdesc_sw128(sbase + P_OFF_K + koff, 16, 1024), id, ks > 0);
        }
        mma_commit(bar_mma);
    }
    GDR_WAIT(bar_mma, ph_mma);
    tc_fence_after();

    // ---- A (fp32, strict lower) and its transposed 16 x 16 diagonal blocks ----
    if ((warp & 3) < 2) {
        const int r = row;  // 0..63
        float d[32];
        tmem_ld32(tmem + lane_base + P_TM_D1 + wg * 32, d);
        const float rf = s_rowf[r] * s_beta[r];
        float* A32 = reinterpret_cast<float*>(sm + P_OFF_A32);
#pragma unroll
        for (int j4 = 0; j4 < 32; j4 += 4) {
            const int j = wg * 32 + j4;
            const float4 c4v = *reinterpret_cast<const float4*>(s_colf + j);
            float4 x;
            x.x = j < r ? rf * c4v.x * d[j4] : 0.f;
            x.y = j + 1 < r ? rf * c4v.y * d[j4 + 1] : 0.f;
            x.z = j + 2 < r ? rf * c4v.z * d[j4 + 2] : 0.f;
            x.w = j + 3 < r ? rf * c4v.w * d[j4 + 3] : 0.f;
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
    }
    __syncthreads();

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
    __syncthreads();

    // ---- D2 = L K (-> W), D3 = PRE V (-> P) --------------------------------------
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idW = idesc_bf16(128, 128, 0, 1);
        const uint32_t idP = idesc_bf16(128, dv, 0, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            mma_bf16(tmem + P_TM_D2, sdesc_sw128(sbase + P_OFF_A32 + ks * 32u, 16, 1024),
                     sdesc_sw128(sbase + P_OFF_K + ks * 2048u, 8192, 1024), idW, ks > 0);
            mma_bf16(tmem + P_TM_D3, sdesc_sw128(sbase + P_OFF_A32 + 8192 + ks * 32u, 16, 1024),
                     sdesc_sw128(sbase + P_OFF_V + ks * 2048u, 8192, 1024), idP, ks > 0);
        }
        mma_commit(bar_mma);
    }
    GDR_WAIT(bar_mma, ph_mma);
    tc_fence_after();

    // ---- rows of -W and P -> workspace (rows 0..63; each warpgroup half the columns)
    if ((warp & 3) < 2) {
        const int r = row;
        const bool valid = r < n;
        const size_t tok = ((size_t)bb * T + t0 + r) * H + h;
        float d[32], d1[32];
        tmem_ld32_async(tmem + lane_base + P_TM_D2 + wg * 64, d);
        tmem_ld32_async(tmem + lane_base + P_TM_D2 + wg * 64 + 32, d1);
        tmem_wait_ld();
        if (valid) {
            __nv_bfloat16* wp = pp.wneg + tok * DK + wg * 64;
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                const float* dd = c8 < 4 ? d + c8 * 8 : d1 + (c8 - 4) * 8;
                uint4 u;
                u.x = pack_bf16x2(-dd[0], -dd[1]);
                u.y = pack_bf16x2(-dd[2], -dd[3]);
                u.z = pack_bf16x2(-dd[4], -dd[5]);
                u.w = pack_bf16x2(-dd[6], -dd[7]);
                *reinterpret_cast<uint4*>(wp + c8 * 8) = u;
            }
        }
        // P: each warpgroup dv / 2 columns (32 or 64)
        const int half = dv >> 1;
        tmem_ld32_async(tmem + lane_base + P_TM_D3 + wg * half, d);
        if (half == 64) tmem_ld32_async(tmem + lane_base + P_TM_D3 + wg * half + 32, d1);
        tmem_wait_ld();
        if (valid) {
            __nv_bfloat16* pq = pp.p + tok * dv + wg * half;
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                if (c8 * 8 >= half) break;
                const float* dd = c8 < 4 ? d + c8 * 8 : d1 + (c8 - 4) * 8;
                uint4 u;
                u.x = pack_bf16x2(dd[0], dd[1]);
                u.y = pack_bf16x2(dd[2], dd[3]);
                u.z = pack_bf16x2(dd[4], dd[5]);
                u.w = pack_bf16x2(dd[6], dd[7]);
                *reinterpret_cast<uint4*>(pq + c8 * 8) = u;
            }
        }
    }

finish:
    if (!ok && tid == 0) flag_status(pp.d_status, GDR_DEVICE_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, P_TM_COLS);
#undef GDR_WAIT
}

// ---- pass 2 shared memory ---------------------------------------------------
constexpr uint32_t S_OFF_WQ = 0;        // [-W ; Q] bf16 [128 x 128], 2 buffers (32 KB each)
constexpr uint32_t S_OFF_K = 65536;     // K bf16 [64 x 128], 2 buffers (B operand of Q K^T)
constexpr uint32_t S_OFF_K2 = 98304;    // K bf16 [64 x 128], 2 buffers, scaled by g_{n-1}/g per token
constexpr uint32_t S_OFF_P = 131072;    // P slice bf16 [64 x 64], 2 buffers
constexpr uint32_t S_OFF_AQ = 147456;   // [0 ; Aq] bf16 [128 x 64]
constexpr uint32_t S_OFF_SBF = 163840;  // S bf16 [128 x 64]
constexpr uint32_t S_OFF_U = 180224;    // U bf16 [64 x 64]
constexpr uint32_t S_OFF_SMALL = 188416;
constexpr uint32_t S_SMEM_BYTES = S_OFF_SMALL + 3072 + 1024;
constexpr uint32_t S_TM_D1 = 0, S_TM_D3 = 64, S_TM_D4 = 128, S_TM_D5 = 192, S_TM_COLS = 256;

__global__ void __launch_bounds__(NT, 1) state_gdn_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_p,
    const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int wg = warp >> 2;
    const int row = tid & 127;
    const int vt = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int v0 = vt * NV;
    const int T = p.T, H = p.H;
    const int nchunks = (T + C - 1) / C;

    // per-token factors, double-buffered by chunk parity: [2][64] each
    float* s_rowf2 = reinterpret_cast<float*>(sm + S_OFF_SMALL);
    float* s_colf2 = s_rowf2 + 128;
    float* s_g2 = s_rowf2 + 256;
    float* s_gcr2 = s_rowf2 + 384;
    float* s_misc2 = s_rowf2 + 512;   // [2][4]: g_{n-1}
    float* s_alpha = s_rowf2 + 520;   // [64] staging of the next chunk's decays
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + S_OFF_SMALL + 2880);  // [2]
    uint64_t* bar_mma = bar_tma + 2;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + S_OFF_SMALL + 2912);
    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_w);
        prefetch_tmap(&tm_p);
    }
    if (warp == 0) tmem_alloc(s_tmem, S_TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t ph_tma0 = 0u, ph_tma1 = 0u, ph_mma = 0;
    bool ok = true;
    const uint32_t sbase = smem_u32(sm);

    auto issue_loads = [&](int ci) {
        const int t0 = ci * C, buf = ci & 1;
        uint8_t* wq = sm + S_OFF_WQ + buf * 32768;
        uint8_t* kk = sm + S_OFF_K + buf * 16384;
        uint8_t* k2 = sm + S_OFF_K2 + buf * 16384;
        mbar_expect_tx(&bar_tma[buf], 9u * 8192u);
        // [-W ; Q]: each 64-column block holds 128 rows (-W rows 0..63, q rows 64..127)
        tma_load_4d(wq, &tm_w, &bar_tma[buf], 0, h, t0, bb);
        tma_load_4d(wq + 16384, &tm_w, &bar_tma[buf], 64, h, t0, bb);
        tma_load_4d(wq + 8192, &tm_q, &bar_tma[buf], 0, h, t0, bb);
        tma_load_4d(wq + 16384 + 8192, &tm_q, &bar_tma[buf], 64, h, t0, bb);
        tma_load_4d(kk, &tm_k, &bar_tma[buf], 0, h, t0, bb);
        tma_load_4d(kk + 8192, &tm_k, &bar_tma[buf], 64, h, t0, bb);
        tma_load_4d(k2, &tm_k, &bar_tma[buf], 0, h, t0, bb);
        tma_load_4d(k2 + 8192, &tm_k, &bar_tma[buf], 64, h, t0, bb);
        tma_load_4d(sm + S_OFF_P + buf * 8192, &tm_p, &bar_tma[buf], v0, h, t0, bb);
    };

    constexpr int NH = NV / 2;
    float S[NH];
    {
        const float* s0 = p.S0 ? p.S0 + (((size_t)bb * H + h) * DK + row) * p.dv + v0 + wg * NH : nullptr;
#pragma unroll
        for (int j = 0; j < NH; j += 4) {
            float4 x = s0 ? *reinterpret_cast<const float4*>(s0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) st_chunk(sm + S_OFF_SBF, sw128_chunk(row, wg * 4 + ch, DK), &S[8 * ch]);
        if (tid < 64) {  // AQ rows 0..63 stay zero
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_zero_chunk(sm + S_OFF_AQ, sw128_chunk(tid, ch, 128));
        }
    }
    unsigned short g_a = 0;
    auto load_alpha = [&](int ci) {
        if (tid < C) {
            const int t = min(ci * C + tid, T - 1);
            g_a = ((const unsigned short*)p.alpha)[((size_t)bb * T + t) * H + h];
        }
    };
    auto bits_to_f32 = [](unsigned short u) { return __uint_as_float((uint32_t)u << 16); };
    auto decay_scan = [&](int ci, int lane) {
        const int par = ci & 1;
        const int n = min(C, T - ci * C);
        const float la0 = (2 * lane < n) ? lg2_approx(s_alpha[2 * lane]) : 0.f;
        const float la1 = (2 * lane + 1 < n) ? lg2_approx(s_alpha[2 * lane + 1]) : 0.f;
        float x = la0 + la1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        const float l1 = x, l0v = x - la1;
        const float first = __shfl_sync(0xffffffffu, l0v, 0);
        const float last = __shfl_sync(0xffffffffu, l1, 31);
        const float ref = 0.5f * (first + last);
        float* rf = s_rowf2 + par * 64;
        float* cf = s_colf2 + par * 64;
        float* g = s_g2 + par * 64;
        float* gcr = s_gcr2 + par * 64;
        rf[2 * lane] = ex2_approx(l0v - ref);
        rf[2 * lane + 1] = ex2_approx(l1 - ref);
        cf[2 * lane] = ex2_approx(ref - l0v);
        cf[2 * lane + 1] = ex2_approx(ref - l1);
        g[2 * lane] = ex2_approx(l0v);
        g[2 * lane + 1] = ex2_approx(l1);
        gcr[2 * lane] = ex2_approx(last - l0v);
        gcr[2 * lane + 1] = ex2_approx(last - l1);
        if (lane == 0) {
            s_misc2[par * 4] = ex2_approx(last);
            if (first - last > 230.f) flag_status(p.d_status, GDR_DEVICE_DECAY_RANGE);
        }
    };
    auto stage_alpha = [&](int ci) {
        if (tid < C) s_alpha[tid] = ci * C + tid < T ? bits_to_f32(g_a) : 1.f;
    };
    if (tid == 0 && nchunks > 0) issue_loads(0);
    if (nchunks > 0) {
        load_alpha(0);
        stage_alpha(0);
        __syncthreads();
        if (warp == 7) decay_scan(0, tid & 31);
        __syncthreads();
    }

#define GDR_WAIT(bar, ph)                                                   \
    do {                                                                    \
        bool w_ok = mbar_wait(bar, ph);                                     \
        ph ^= 1u;                                                           \
        if (!__syncthreads_and(w_ok)) { ok = false; goto finish; }          \
    } while (0)
#define GDR_BEFORE_MMA()    \
    do {                    \
        fence_proxy_async(); \
        tc_fence_before();  \
        __syncthreads();    \
    } while (0)

    for (int ci = 0; ci < nchunks; ++ci) {
        const int t0 = ci * C;
        const int buf = ci & 1;
        const uint32_t wqb = sbase + S_OFF_WQ + buf * 32768u;
        const uint32_t kb = sbase + S_OFF_K + buf * 16384u;
        const uint32_t k2b = sbase + S_OFF_K2 + buf * 16384u;
        if (tid == 0 && ci + 1 < nchunks) issue_loads(ci + 1);  // its buffers were freed by chunk ci-1
        if (ci + 1 < nchunks) load_alpha(ci + 1);
        const int par = ci & 1;
        const float* s_rowf = s_rowf2 + par * 64;
        const float* s_colf = s_colf2 + par * 64;
        const float* s_g = s_g2 + par * 64;
        const float* s_gcr = s_gcr2 + par * 64;
        const float* s_misc = s_misc2 + par * 4;
        if (buf == 0) GDR_WAIT(&bar_tma[0], ph_tma0);
        else GDR_WAIT(&bar_tma[1], ph_tma1);

        // ---- batch 1: D3 = [-W ; Q] S;  D1 = [-W ; Q] K^T (rows 64..127: Q K^T) ------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idS = idesc_bf16(128, NV, 0, 1);
            const uint32_t idK = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t koff = (ks >> 2) * 16384u + (ks & 3) * 32u;
                const uint32_t kkoff = (ks >> 2) * 8192u + (ks & 3) * 32u;
                mma_bf16(tmem + S_TM_D3, sdesc_sw128(wqb + koff, 16, 1024),
                         sdesc_sw128(sbase + S_OFF_SBF + ks * 2048u, 8192, 1024), idS, ks > 0);
                mma_bf16(tmem + S_TM_D1, sdesc_sw128(wqb + koff, 16, 1024),
                         sdesc_sw128(kb + kkoff, 16, 1024), idK, ks > 0);
            }
            mma_commit(bar_mma);
        }
        // while batch 1 runs: scale the K2 copy's rows by g_{n-1} / g_r
        {
            const int r = tid >> 2, c4 = (tid & 3) * 4;  // 64 rows x 4 threads x 4 chunks
            const float f = s_gcr[r];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float x[8];
                const uint32_t off = sw128_chunk(r, c4 + cc, 64);
                ld_chunk(sm + S_OFF_K2 + buf * 16384, off, x);
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] *= f;
                st_chunk(sm + S_OFF_K2 + buf * 16384, off, x);
            }
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();

        // ---- U = P - W S (rows 0..63) -> bf16;  Aq (rows 64..127) -> [0 ; Aq] -------
        if (row < 64) {
            float d[32];
            tmem_ld32(tmem + lane_base + S_TM_D3 + wg * 32, d);
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                float x[8];
                ld_chunk(sm + S_OFF_P + buf * 8192, sw128_chunk(row, wg * 4 + c8, 64), x);
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] += d[c8 * 8 + e];
                st_chunk(sm + S_OFF_U, sw128_chunk(row, wg * 4 + c8, 64), x);
            }
        } else {
            const int r = row - 64;
            float d[32];
            tmem_ld32(tmem + lane_base + S_TM_D1 + wg * 32, d);
            const float rf = s_rowf[r];
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                float x[8];
                const float4 ca = *reinterpret_cast<const float4*>(s_colf + wg * 32 + c8 * 8);
                const float4 cb = *reinterpret_cast<const float4*>(s_colf + wg * 32 + c8 * 8 + 4);
                const float cf[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j = wg * 32 + c8 * 8 + e;
                    x[e] = j <= r ? rf * cf[e] * d[c8 * 8 + e] : 0.f;
                }
                st_chunk(sm + S_OFF_AQ, sw128_chunk(row, wg * 4 + c8, 128), x);
            }
        }
        if (ci + 1 < nchunks) stage_alpha(ci + 1);
        GDR_BEFORE_MMA();

        // ---- batch 2: D5 = [0 ; Aq] U;  D4 = (Diag(g_{n-1}/g) K)^T U ------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idK = idesc_bf16(128, NV, 0, 1);
            const uint32_t idM = idesc_bf16(128, NV, 1, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                mma_bf16(tmem + S_TM_D5, sdesc_sw128(sbase + S_OFF_AQ + ks * 32u, 16, 1024),
                         sdesc_sw128(sbase + S_OFF_U + ks * 2048u, 8192, 1024), idK, ks > 0);
                mma_bf16(tmem + S_TM_D4, sdesc_sw128(k2b + ks * 2048u, 8192, 1024),
                         sdesc_sw128(sbase + S_OFF_U + ks * 2048u, 8192, 1024), idM, ks > 0);
            }
            mma_commit(bar_mma);
        }
        if (warp == 7 && ci + 1 < nchunks) decay_scan(ci + 1, tid & 31);  // overlaps batch 2
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();

        // ---- O = g Q S + Aq U (rows 64..127) -> global; S = g_{n-1} S + D4 ----------
        {
            float d[32], d5[32], dS[32];
            if (row >= 64) {
                tmem_ld32_async(tmem + lane_base + S_TM_D3 + wg * 32, d);
                tmem_ld32_async(tmem + lane_base + S_TM_D5 + wg * 32, d5);
            }
            tmem_ld32_async(tmem + lane_base + S_TM_D4 + wg * 32, dS);
            tmem_wait_ld();
            if (row >= 64) {
                const int t = t0 + row - 64;
                if (t < T) {
                    const float gr = s_g[row - 64];
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
            }
            const float gC = s_misc[0];
#pragma unroll
            for (int j = 0; j < NH; ++j) S[j] = fmaf(gC, S[j], dS[j]);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) st_chunk(sm + S_OFF_SBF, sw128_chunk(row, wg * 4 + ch, DK), &S[8 * ch]);
        }
        tc_fence_before();
        __syncthreads();
    }

    if (p.ST) {
        float* st = p.ST + (((size_t)bb * H + h) * DK + row) * p.dv + v0 + wg * NH;
#pragma unroll
        for (int j = 0; j < NH; j += 4) *reinterpret_cast<float4*>(st + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }

finish:
    if (!ok && tid == 0) flag_status(p.d_status, GDR_DEVICE_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, S_TM_COLS);
#undef GDR_WAIT
#undef GDR_BEFORE_MMA
}

}  // namespace twopass

size_t twopass_workspace_bytes(int B, int T, int H, int dv) {
    return (size_t)B * T * H * (chunkc::DK + dv) * sizeof(__nv_bfloat16);
}

// maps: q, k, v, then the workspace maps -W ([B,T,H,128]) and P ([B,T,H,d_v]).
cudaError_t launch_chunk_twopass_gdn(const CUtensorMap* maps, const CUtensorMap* ws_maps, void* ws,
                                     const void* alpha, const void* beta, const float* S0, void* o,
                                     float* ST, int* d_status, int B, int T, int H, int dv,
                                     cudaStream_t st) {
    using namespace twopass;
    PrepParams pp;
    pp.alpha = alpha; pp.beta = beta;
    pp.wneg = reinterpret_cast<__nv_bfloat16*>(ws);
    pp.p = reinterpret_cast<__nv_bfloat16*>(ws) + (size_t)B * T * H * DK;
    pp.d_status = d_status;
    pp.T = T; pp.H = H; pp.dv = dv;
    cudaError_t e = cudaFuncSetAttribute(prep_gdn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int nchunks = (T + C - 1) / C;
    prep_gdn_kernel<<<dim3(nchunks, H, B), NT, P_SMEM_BYTES, st>>>(maps[1], maps[2], pp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    Params p;
    p.alpha = alpha; p.bg = beta; p.wg = nullptr;
    p.S0 = S0; p.o = (__nv_bfloat16*)o; p.ST = ST; p.d_status = d_status;
    p.B = B; p.T = T; p.H = H; p.dv = dv;
    p.akind = GDR_GATE_SCALAR; p.bkind = GDR_GATE_SCALAR; p.wkind = GDR_GATE_TIED;
    e = cudaFuncSetAttribute(state_gdn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, S_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    state_gdn_kernel<<<dim3(dv / NV, H, B), NT, S_SMEM_BYTES, st>>>(maps[0], maps[1], ws_maps[0], ws_maps[1], p);
    return cudaGetLastError();
}

}  // namespace gdr
