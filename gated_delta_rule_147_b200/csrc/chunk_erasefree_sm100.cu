// Erase-free chunkwise forward (b = 0) on sm_100a tensor cores: linear
// attention (alpha = 1), gated linear attention / Mamba-2 shapes (scalar or
// channel-wise decay), with an optional write gate w.
//
// Without erase the recurrence is S_t = Diag(alpha_t) S_{t-1} + (w_t.k_t)^T v_t
// ("Recurrent Memory: Write, Erase, Decay, Read", sections 01 and 04; the
// structured masked-matrix reading of "The Eraser Trilogy", "The Rosetta
// Stone"). Per chunk of C = 64 tokens, with l_r the prefix sum of log2 alpha,
// rowf_r = 2^(l_r - ref), colf_r = 2^(ref - l_r) and g_r = 2^l_r:
//   Bq = lower[(q.rowf)(w.k.colf)^T]                  (decay-masked q k^T)
//   O  = (q.g) S + Bq V
//   S' = Diag(g_{n-1}) S + Diag(2^(l_{n-1}-ref)) (w.k.colf)^T V
// No triangular solve and no per-chunk "new values": three independent
// MMAs issue in one batch (Bq, (q.g) S, the state increment), one more adds
// Bq V after Bq is masked into bf16.
#include "chunk_common.cuh"

namespace gdr {
namespace erasefree {

using namespace chunkc;

constexpr uint32_t OFF_QIN = 0;        // q [64 x 128] bf16 (TMA)
constexpr uint32_t OFF_KIN = 16384;    // k
constexpr uint32_t OFF_GA = 32768;     // channel alpha
constexpr uint32_t OFF_GW = 49152;     // channel w
constexpr uint32_t OFF_AQG = 65536;    // [q.g ; q.rowf] bf16 [128 x 128]
constexpr uint32_t OFF_KWS = 98304;    // w.k.colf bf16 [64 x 128]
constexpr uint32_t OFF_BQ = 114688;    // [Bq ; 0] bf16 [128 x 64]
constexpr uint32_t OFF_V = 131072;     // v slice [64 x NVT] bf16 (NVT / 64 tiles of 8 KB), two buffers
// The CTA's value columns NVT (64 or 128; 128 halves the CTA count where there
// are more 64-column tiles than SMs) size the rest of the map:
template <int NVT>
struct Lay {
    static constexpr uint32_t VBUF = NVT / 64 * 8192;          // one V buffer
    static constexpr uint32_t SBF = OFF_V + 2 * VBUF;          // S bf16 [128 x NVT] (16 KB per 64 columns)
    static constexpr uint32_t SCAN = SBF + NVT / 64 * 16384;   // scan scratch fp32 [9 x 128]
    static constexpr uint32_t SMALL = SCAN + 6144;             // scalars, barriers
    static constexpr uint32_t BYTES = SMALL + 3072 + 1024;
    static constexpr uint32_t TM_D1 = 0, TM_D3 = 64, TM_D4 = 64 + NVT;
    static constexpr uint32_t TM_COLS = NVT == 64 ? 256 : 512;
};

template <bool ACH, int NVT>
__global__ void __launch_bounds__(NT, 1) chunk_fwd_erasefree_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
    const __grid_constant__ CUtensorMap tm_w, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, wg = warp >> 2, row = tid & 127;
    const int vt = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int hq = h / p.group;  // q / k head of this value head
    const int v0 = vt * NVT;
    using L = Lay<NVT>;
    constexpr uint32_t OFF_SBF = L::SBF, OFF_SCAN = L::SCAN, OFF_SMALL = L::SMALL;
    constexpr uint32_t TM_D1 = L::TM_D1, TM_D3 = L::TM_D3, TM_D4 = L::TM_D4, TM_COLS = L::TM_COLS;
    const int T = p.T, H = p.H;
    const int nchunks = (T + C - 1) / C;
    const bool wch = p.wkind == GDR_GATE_CHANNEL;

    float* s_a = reinterpret_cast<float*>(sm + OFF_SMALL);  // [64] scalar alpha
    float* s_w = s_a + 64;                                  // [64] scalar w
    float* s_rowf = s_a + 128;                              // [64] scalar decay
    float* s_colf = s_a + 192;                              // [64]
    float* s_eref = s_a + 256;                              // [128] 2^ref
    float* s_gC = s_a + 384;                                // [128]
    float* s_fS = s_a + 512;                                // [128]
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + OFF_SMALL + 2560);
    uint64_t* bar_mma = bar_tma + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + OFF_SMALL + 2576);

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) tmem_alloc(s_tmem, TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t ph_tma = 0, ph_mma = 0;
    bool ok = true;
    const uint32_t sbase = smem_u32(sm);

    auto issue_loads = [&](int ci) {
        const int t0 = ci * C;
        mbar_expect_tx(bar_tma, (uint32_t)(4 + NVT / 64 + 2 * (ACH + wch)) * 8192u);
        tma_load_4d(sm + OFF_QIN, &tm_q, bar_tma, 0, hq, t0, bb);
        tma_load_4d(sm + OFF_QIN + 8192, &tm_q, bar_tma, 64, hq, t0, bb);
        tma_load_4d(sm + OFF_KIN, &tm_k, bar_tma, 0, hq, t0, bb);
        tma_load_4d(sm + OFF_KIN + 8192, &tm_k, bar_tma, 64, hq, t0, bb);
#pragma unroll
        for (int i = 0; i < NVT / 64; ++i)
            tma_load_4d(sm + OFF_V + (ci & 1) * L::VBUF + i * 8192, &tm_v, bar_tma, v0 + 64 * i, h, t0, bb);
        if (ACH) {
            tma_load_4d(sm + OFF_GA, &tm_a, bar_tma, 0, h, t0, bb);
            tma_load_4d(sm + OFF_GA + 8192, &tm_a, bar_tma, 64, h, t0, bb);
        }
        if (wch) {
            tma_load_4d(sm + OFF_GW, &tm_w, bar_tma, 0, h, t0, bb);
            tma_load_4d(sm + OFF_GW + 8192, &tm_w, bar_tma, 64, h, t0, bb);
        }
    };

    constexpr int NH = NVT / 2;
    float S[NH];
    {
        const float* s0 = p.S0 ? p.S0 + (((size_t)bb * H + h) * DK + row) * p.dv + v0 + wg * NH : nullptr;
#pragma unroll
        for (int j = 0; j < NH; j += 4) {
            float4 x = s0 ? *reinterpret_cast<const float4*>(s0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
#pragma unroll
        for (int ch = 0; ch < NH / 8; ++ch) st_chunk(sm + OFF_SBF, sw128_chunk(row, wg * (NH / 8) + ch, DK), &S[8 * ch]);
        if (tid < 64) {  // rows 64..127 of [Bq ; 0] stay zero
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_zero_chunk(sm + OFF_BQ, sw128_chunk(64 + tid, ch, 128));
        }
    }
    unsigned short g_a = 0, g_w = 0;
    auto load_scalar_gates = [&](int ci) {
        if (tid < C) {
            const int t = min(ci * C + tid, T - 1);
            const size_t gi = ((size_t)bb * T + t) * H + h;
            if (p.akind == GDR_GATE_SCALAR) g_a = ((const unsigned short*)p.alpha)[gi];
            if (p.wkind == GDR_GATE_SCALAR) g_w = ((const unsigned short*)p.wg)[gi];
        }
    };
    auto bits_to_f32 = [](unsigned short u) { return __uint_as_float((uint32_t)u << 16); };
    if (tid == 0 && nchunks > 0) issue_loads(0);
    if (nchunks > 0) load_scalar_gates(0);

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
        const int n = min(C, T - t0);
        const uint32_t vbuf = sbase + OFF_V + (ci & 1) * L::VBUF;
        if (tid < C) {
            const bool valid = t0 + tid < T;
            s_a[tid] = (p.akind == GDR_GATE_SCALAR && valid) ? bits_to_f32(g_a) : 1.f;
            s_w[tid] = (p.wkind == GDR_GATE_SCALAR && valid) ? bits_to_f32(g_w)
                       : (p.wkind == GDR_GATE_NONE ? 1.f : 0.f);
        }
        GDR_WAIT(bar_tma, ph_tma);
        if (ci + 1 < nchunks) load_scalar_gates(ci + 1);

        // ---- build: decay scan, [q.g ; q.rowf] and w.k.colf -----------------------
        {
            const int cg = tid & 31, rg = warp;  // 8 tokens x 4 channels per thread
            const int ch0 = cg * 4;
            float* scan = reinterpret_cast<float*>(sm + OFF_SCAN);
            bool chunk_bad = false;  // decay span beyond the factorisation's range
            float lrow[8][4], aval[8][4];
            if (!ACH) {
                if (warp == 0) {
                    const int lane = tid;
                    const float la0 = (2 * lane < n) ? lg2_approx(s_a[2 * lane]) : 0.f;
                    const float la1 = (2 * lane + 1 < n) ? lg2_approx(s_a[2 * lane + 1]) : 0.f;
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
                    if (lane == 0) {
                        scan[0] = ex2_approx(ref);
                        scan[1] = ex2_approx(last);
                        scan[2] = ex2_approx(last - ref);
                        scan[3] = first - last > 230.f ? 1.f : 0.f;
                    }
                }
                __syncthreads();
                chunk_bad = scan[3] != 0.f;
                if (tid < 128) {
                    s_eref[tid] = scan[0];
                    s_gC[tid] = scan[1];
                    s_fS[tid] = scan[2];
                }
            } else {
                float loc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = rg * 8 + i;
                    ld4(sm + OFF_GA, piece4(r, cg, C), aval[i]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if (r >= n) aval[i][e] = 1.f;
                        loc[e] += lg2_approx(aval[i][e]);
                        lrow[i][e] = loc[e];
                    }
                }
                *reinterpret_cast<float4*>(scan + rg * 128 + ch0) = make_float4(loc[0], loc[1], loc[2], loc[3]);
                if (rg == 0)
                    *reinterpret_cast<float4*>(scan + 1024 + ch0) =
                        make_float4(lrow[0][0], lrow[0][1], lrow[0][2], lrow[0][3]);
                __syncthreads();
                float pre[4] = {0.f, 0.f, 0.f, 0.f}, tot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const float4 x = *reinterpret_cast<const float4*>(scan + g * 128 + ch0);
                    const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if (g < rg) pre[e] += xs[e];
                        tot[e] += xs[e];
                    }
                }
                const float4 l04 = *reinterpret_cast<const float4*>(scan + 1024 + ch0);
                const float l0[4] = {l04.x, l04.y, l04.z, l04.w};
                bool bad = false;
                float ref[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    ref[e] = 0.5f * (l0[e] + tot[e]);
                    bad |= (l0[e] - tot[e]) > 230.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) lrow[i][e] += pre[e] - ref[e];
                }
                chunk_bad = bad;
                if (rg == 0) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        s_eref[ch0 + e] = ex2_approx(ref[e]);
                        s_gC[ch0 + e] = ex2_approx(tot[e]);
                        s_fS[ch0 + e] = ex2_approx(tot[e] - ref[e]);
                    }
                }
                __syncthreads();  // s_eref of every channel is needed below
            }
            if (__syncthreads_or(chunk_bad)) {
                // the chunk's decay ratios do not fit two bounded factors: apply
                // its tokens one by one (fp32, raw inputs), then go on
                if (tid == 0) flag_status(p.d_status, GDR_DEVICE_DECAY_RANGE);
                if (tid == 0 && ci + 1 < nchunks) issue_loads(ci + 1);
                const ExactArgs ex{(const __nv_bfloat16*)p.q, (const __nv_bfloat16*)p.k,
                                   (const __nv_bfloat16*)p.v, (const __nv_bfloat16*)p.alpha,
                                   nullptr, (const __nv_bfloat16*)p.wg,
                                   p.akind, GDR_GATE_NONE, p.wkind, p.o, T, H, H / p.group, p.dv};
                exact_tokens(ex, S, scan, bb, h, hq, v0, t0, n, tid);
#pragma unroll
                for (int ch = 0; ch < NH / 8; ++ch)
                    st_chunk(sm + OFF_SBF, sw128_chunk(row, wg * (NH / 8) + ch, DK), &S[8 * ch]);
                fence_proxy_async();
                tc_fence_before();
                __syncthreads();
                continue;
            }
            float er[4];
            if (ACH) {
                const float4 e4 = *reinterpret_cast<const float4*>(s_eref + ch0);
                er[0] = e4.x; er[1] = e4.y; er[2] = e4.z; er[3] = e4.w;
            } else {
                er[0] = er[1] = er[2] = er[3] = scan[0];  // one decay per token: uniform 2^ref
            }
            float rowf_c[4];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = rg * 8 + i;
                float k4[4], q4[4], w4[4];
                ld4(sm + OFF_KIN, piece4(r, cg, C), k4);
                ld4(sm + OFF_QIN, piece4(r, cg, C), q4);
                if (wch) ld4(sm + OFF_GW, piece4(r, cg, C), w4);
                else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) w4[e] = s_w[r];
                }
                const bool valid = r < n;
                const float rs = ACH ? 0.f : s_rowf[r], cs = ACH ? 0.f : s_colf[r];
                if (ACH) {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        rowf_c[e] = (i == 0) ? ex2_approx(lrow[0][e]) : rowf_c[e] * aval[i][e];
                }
                float qg[4], qs[4], kw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float rowf = ACH ? rowf_c[e] : rs;
                    const float colf = ACH ? rcp_newton(rowf) : cs;
                    const float kk = valid ? k4[e] : 0.f;
                    const float qq = valid ? q4[e] : 0.f;
                    qs[e] = qq * rowf;
                    qg[e] = qs[e] * er[e];
                    kw[e] = w4[e] * kk * colf;
                }
                st4(sm, OFF_AQG + piece4(r, cg, 128), qg);
                st4(sm, OFF_AQG + piece4(64 + r, cg, 128), qs);
                st4(sm, OFF_KWS + piece4(r, cg, C), kw);
            }
        }
        GDR_BEFORE_MMA();
        // the input tiles are consumed: prefetch the next chunk (its v buffer was
        // last read by the previous chunk's MMAs, which completed)
        if (tid == 0 && ci + 1 < nchunks) issue_loads(ci + 1);

        // ---- one batch: Bq raw, (q.g) S, state increment ------------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id64 = idesc_bf16(128, 64, 0, 0);
            const uint32_t idS = idesc_bf16(128, NVT, 0, 1);
            const uint32_t idM = idesc_bf16(128, NVT, 1, 1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t koff = (ks >> 2) * 16384u + (ks & 3) * 32u;
                const uint32_t koffk = (ks >> 2) * 8192u + (ks & 3) * 32u;
                mma_bf16(tmem + TM_D1, sdesc_sw128(sbase + OFF_AQG + koff, 16, 1024),
                         sdesc_sw128(sbase + OFF_KWS + koffk, 16, 1024), id64, ks > 0);
                mma_bf16(tmem + TM_D3, sdesc_sw128(sbase + OFF_AQG + koff, 16, 1024),
                         sdesc_sw128(sbase + OFF_SBF + ks * 2048u, 16384, 1024), idS, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + TM_D4, sdesc_sw128(sbase + OFF_KWS + ks * 2048u, 8192, 1024),
                         sdesc_sw128(vbuf + ks * 2048u, 8192, 1024), idM, ks > 0);
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();

        // ---- Bq: rows 64..127 of D1 masked to j <= r -> rows 0..63 of [Bq ; 0] ------
        if (row >= 64) {
            const int r = row - 64;
            float d[32];
            tmem_ld32(tmem + lane_base + TM_D1 + wg * 32, d);
            float x[8];
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = (wg * 32 + c8 * 8 + e <= r) ? d[c8 * 8 + e] : 0.f;
                st_chunk(sm + OFF_BQ, sw128_chunk(r, wg * 4 + c8, 128), x);
            }
        }
        GDR_BEFORE_MMA();

        // ---- O += Bq V -------------------------------------------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idS = idesc_bf16(128, NVT, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + TM_D3, sdesc_sw128(sbase + OFF_BQ + ks * 32u, 16, 1024),
                         sdesc_sw128(vbuf + ks * 2048u, 8192, 1024), idS, 1);
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();

        // ---- O (rows 0..63 of D3) -> global; S = g S + f D4 (32 columns at a time) ----
        {
            const float gC = s_gC[row], fS = s_fS[row];
#pragma unroll
            for (int hf = 0; hf < NH / 32; ++hf) {
                float d[32], dS[32];
                const uint32_t col = wg * NH + hf * 32;
                if (row < 64) tmem_ld32_async(tmem + lane_base + TM_D3 + col, d);
                tmem_ld32_async(tmem + lane_base + TM_D4 + col, dS);
                tmem_wait_ld();
                if (row < 64) {
                    const int t = t0 + row;
                    if (t < T) {
                        __nv_bfloat16* op = p.o + (((size_t)bb * T + t) * H + h) * p.dv + v0 + col;
#pragma unroll
                        for (int c8 = 0; c8 < 4; ++c8) {
                            uint4 u;
                            u.x = pack_bf16x2(d[c8 * 8 + 0], d[c8 * 8 + 1]);
                            u.y = pack_bf16x2(d[c8 * 8 + 2], d[c8 * 8 + 3]);
                            u.z = pack_bf16x2(d[c8 * 8 + 4], d[c8 * 8 + 5]);
                            u.w = pack_bf16x2(d[c8 * 8 + 6], d[c8 * 8 + 7]);
                            *reinterpret_cast<uint4*>(op + c8 * 8) = u;
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) S[hf * 32 + j] = gC * S[hf * 32 + j] + fS * dS[j];
            }
#pragma unroll
            for (int ch = 0; ch < NH / 8; ++ch) st_chunk(sm + OFF_SBF, sw128_chunk(row, wg * (NH / 8) + ch, DK), &S[8 * ch]);
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
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
#undef GDR_WAIT
#undef GDR_BEFORE_MMA
}

}  // namespace erasefree

// maps: q, k, v, alpha (channel) or q, w (channel) or q
cudaError_t launch_chunk_erasefree_sm100(const CUtensorMap* maps, const void* q, const void* k,
                                         const void* v, const void* alpha, const void* w,
                                         int akind, int wkind, const float* S0, void* o, float* ST,
                                         int* d_status, int B, int T, int H, int dv, int group,
                                         cudaStream_t st) {
    chunkc::Params p;
    p.q = q; p.k = k; p.v = v;
    p.alpha = alpha; p.bg = nullptr; p.wg = w;
    p.S0 = S0; p.o = (__nv_bfloat16*)o; p.ST = ST; p.d_status = d_status;
    p.B = B; p.T = T; p.H = H; p.dv = dv;
    p.akind = akind; p.bkind = GDR_GATE_NONE; p.wkind = wkind;
    p.group = group;
    // 128 value columns per CTA when there are more 64-column tiles than SMs
    // (one wave instead of two); the MMAs cost the same to issue at N = 128
    int dev = 0, nsm = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 == cudaSuccess) e0 = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e0 != cudaSuccess) return e0;
    const bool wide = dv % 128 == 0 && (long long)(dv / 64) * H * B > nsm;
    auto launch = [&](auto kern, int nvt, uint32_t bytes) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        kern<<<dim3(dv / nvt, H, B), chunkc::NT, bytes, st>>>(maps[0], maps[1], maps[2], maps[3], maps[5], p);
        return cudaGetLastError();
    };
    using namespace erasefree;
    if (wide)
        return akind == GDR_GATE_CHANNEL ? launch(chunk_fwd_erasefree_kernel<true, 128>, 128, Lay<128>::BYTES)
                                         : launch(chunk_fwd_erasefree_kernel<false, 128>, 128, Lay<128>::BYTES);
    return akind == GDR_GATE_CHANNEL ? launch(chunk_fwd_erasefree_kernel<true, 64>, 64, Lay<64>::BYTES)
                                     : launch(chunk_fwd_erasefree_kernel<false, 64>, 64, Lay<64>::BYTES);
}

}  // namespace gdr
