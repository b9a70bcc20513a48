// Two-pass chunkwise forward for channel-wise decay and for independent erase
// / write gates (Kimi Delta Attention and Gated DeltaNet-2 forms) on sm_100a.
//
// Same chunk algebra as the single-pass kernel ("Recurrent Memory: Write,
// Erase, Decay, Read" sections 03-05; "Erase-then-Delta Attention" abstract),
// with l_r the per-channel prefix sum of log2 alpha over the chunk, ref the
// chunk's reference, rowf = 2^(l - ref), colf = 2^(ref - l), g = 2^l:
//   Kb = b.k.rowf   Qs = q.rowf   Ks = k.colf   Kws = w.k.colf
//   A  = strict_lower(Kb Ks^T)    Bm = strict_lower(Kb Kws^T)
//   Aq = lower(Qs Ks^T)           Bq = lower(Qs Kws^T)
//   T  = (I + A)^-1,  W = T Kb . 2^ref
// Everything that does not involve the state is formed in pass 1, one CTA per
// chunk, all chunks of all heads in parallel, into a workspace:
//   WN = -W          QG = q.g               K2 = k.g_{n-1}/g    AQ = Aq
//   P  = T Diag(beta) V (tied beta)  or  -T Bm V (independent gates)
//   KW2 = w.k.g_{n-1}/g,  BQ = Bq    (independent gates only)
//   GC = g_{n-1}  (fp32, per chunk and channel)
// Pass 2 walks the chunks of one (batch, head, 64 columns of d_v) in order:
//   U  = P + WN S
//   O  = QG S + AQ U (+ BQ V)
//   S' = Diag(GC) S + K2^T U (+ KW2^T V)
// With tied beta, Bm = A Diag(beta) and Bq = Aq Diag(beta), so U + Diag(beta) V
// = T Diag(beta) V - W S replaces U and the V terms drop out.
#include <mutex>

#include "chunk_common.cuh"

namespace gdr {
namespace twopass_g {

using namespace chunkc;

// Optional phase tracing (build with -DGDR_TRACE_PHASES): clock64() stamps of
// thread 0 of the pass-1 CTAs of head (0, 0), chunks 0..63 (16 slots each);
// gdr_trace_general_read() copies them out.
#ifdef GDR_TRACE_PHASES
__device__ unsigned long long g_trace3[64 * 16];
#define GDR_TRACE_G(k)                                                                     \
    do {                                                                                  \
        if (blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0 && blockIdx.x < 64)    \
            g_trace3[blockIdx.x * 16 + (k)] = clock64();                                  \
    } while (0)
#else
#define GDR_TRACE_G(k) \
    do {              \
    } while (0)
#endif

// ---- pass 1 shared memory (bytes from a 1024-aligned base) ----------------
// M = 128 MMAs read A rows 64..127 beyond each 64-row operand; those rows
// land in the next region (garbage rows whose outputs are never read).
constexpr uint32_t G_OFF_ROP = 0;       // [Kb ; Qs] bf16 [128 x 128] (two 16 KB column blocks);
                                        // after P1 the Qs rows hold the V tiles
constexpr uint32_t G_OFF_COP = 32768;   // [Ks ; Kws] bf16 [64 | 128 x 128]; after P1: A32, T32
constexpr uint32_t G_OFF_A32 = 32768;   // A fp32 [64 x 64]
constexpr uint32_t G_OFF_T32 = 49152;   // T fp32 [64 x 64]
constexpr uint32_t G_OFF_SCR = 65536;   // decay-scan scratch in the build, solve scratch after (5 KB)
constexpr uint32_t G_OFF_APRE = 71680;  // T Diag(beta) (tied) or -T Bm, bf16 [64 x 64]
constexpr uint32_t G_OFF_L = 79872;     // T bf16 [64 x 64]
constexpr uint32_t G_OFF_X = 88064;     // Bm bf16 [64 x 64]
constexpr uint32_t G_OFF_SMALL = 96256;
constexpr uint32_t G_SMEM_BYTES = G_OFF_SMALL + 3072 + 1024;
constexpr uint32_t G_TM_COLS = 256;

struct GPrepParams {
    int c_begin;  // chunk index of blockIdx.x = 0
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* alpha;
    const __nv_bfloat16* bg;
    const __nv_bfloat16* wg;
    __nv_bfloat16 *wn, *qg, *k2, *kw2, *aq, *bq, *p;  // [B, T, H, d]
    float* gc;                                        // [B, H, nchunks, 128]
    int* d_status;
    int T, H, dv, akind, bkind, wkind;
    int group;  // value heads per q/k head (q, k read at token-head index / group)
    const __nv_bfloat16* v;
    int prefetch_ahead;  // CTAs between this one and the one whose inputs it pulls into L2 (0: none)
};

__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("{\n\t.reg .u64 g;\n\tcvta.to.global.u64 g, %0;\n\tprefetch.global.L2 [g];\n\t}" ::"l"(p));
}

__device__ __forceinline__ void ld8b(const __nv_bfloat16* p, uint2& u) {
    u = *reinterpret_cast<const uint2*>(p);
}
__device__ __forceinline__ void unpack4(const uint2& u, float* x4) {
    const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    x4[0] = f0.x; x4[1] = f0.y; x4[2] = f1.x; x4[3] = f1.y;
}
__device__ __forceinline__ void st8b(__nv_bfloat16* p, const float* x4) {
    uint2 u;
    u.x = pack_bf16x2(x4[0], x4[1]);
    u.y = pack_bf16x2(x4[2], x4[3]);
    *reinterpret_cast<uint2*>(p) = u;
}
// 32 consecutive fp32 values (one thread's TMEM row slice) -> bf16 in global
__device__ __forceinline__ void st32_bf16(__nv_bfloat16* p, const float* x, float sign) {
#pragma unroll
    for (int c8 = 0; c8 < 4; ++c8) {
        uint4 u;
        u.x = pack_bf16x2(sign * x[c8 * 8 + 0], sign * x[c8 * 8 + 1]);
        u.y = pack_bf16x2(sign * x[c8 * 8 + 2], sign * x[c8 * 8 + 3]);
        u.z = pack_bf16x2(sign * x[c8 * 8 + 4], sign * x[c8 * 8 + 5]);
        u.w = pack_bf16x2(sign * x[c8 * 8 + 6], sign * x[c8 * 8 + 7]);
        *reinterpret_cast<uint4*>(p + c8 * 8) = u;
    }
}

template <bool TIED, bool ACH>
__global__ void __launch_bounds__(NT, 2) prep_general_kernel(
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_wn,
    const __grid_constant__ CUtensorMap tm_aq, const __grid_constant__ CUtensorMap tm_p,
    const __grid_constant__ CUtensorMap tm_bq, const GPrepParams pp) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, wg = warp >> 2, row = tid & 127;
    const int ci = pp.c_begin + (int)blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int T = pp.T, H = pp.H, dv = pp.dv;
    const int nchunks = (T + C - 1) / C;
    const int t0 = ci * C;
    const int n = min(C, T - t0);
    const int nvt = dv / 64;
    const bool bch = pp.bkind == GDR_GATE_CHANNEL, wch = pp.wkind == GDR_GATE_CHANNEL;
    constexpr int N1 = TIED ? 64 : 128;  // rows of [Ks ; Kws]
    const int cg = tid & 31, rg = warp;  // build: thread = 8 tokens (rg) x 4 channels (cg)
    const int ch0 = cg * 4;

    // ---- global loads first: scalar gates (raw bf16 bits), channel decay of the
    //      thread's 8 tokens, and q, k, b, w of its first 4 tokens ----------------
    unsigned short g_a = 0, g_b = 0, g_w = 0;
    if (tid < C) {
        const size_t gi = ((size_t)bb * T + t0 + min(tid, n - 1)) * H + h;
        if (pp.akind == GDR_GATE_SCALAR) g_a = reinterpret_cast<const unsigned short*>(pp.alpha)[gi];
        if (pp.bkind == GDR_GATE_SCALAR) g_b = reinterpret_cast<const unsigned short*>(pp.bg)[gi];
        if (pp.wkind == GDR_GATE_SCALAR) g_w = reinterpret_cast<const unsigned short*>(pp.wg)[gi];
    }
    auto elem = [&](int r) {  // element index of (token row r, channel ch0)
        return (((size_t)bb * T + t0 + min(r, n - 1)) * H + h) * DK + ch0;
    };
    const int Hq = H / pp.group, hq = h / pp.group;  // q / k heads; this value head's
    auto elem_qk = [&](int r) {
        return (((size_t)bb * T + t0 + min(r, n - 1)) * Hq + hq) * DK + ch0;
    };
    uint2 aa[8];
    if (ACH) {
#pragma unroll
        for (int i = 0; i < 8; ++i) ld8b(pp.alpha + elem(rg * 8 + i), aa[i]);
    }
    // q, k, b, w of token rg * 8 + i live in slot i % 4: tokens 0..3 now, token
    // i + 4 is loaded into the slot as soon as token i has been unpacked
    uint2 qa[4], ka[4], ba[4], wa[4];
    auto load_token = [&](int i) {
        const size_t e = elem(rg * 8 + i);
        const size_t eq = elem_qk(rg * 8 + i);
        const int sl = i & 3;
        ld8b(pp.q + eq, qa[sl]);
        ld8b(pp.k + eq, ka[sl]);
        if (bch) ld8b(pp.bg + e, ba[sl]);
        if (!TIED && wch) ld8b(pp.wg + e, wa[sl]);
    };
#pragma unroll
    for (int i = 0; i < 4; ++i) load_token(i);

    float* s_ascal = reinterpret_cast<float*>(sm + G_OFF_SMALL);
    float* s_bscal = s_ascal + 64;
    float* s_wscal = s_ascal + 128;
    float* s_rowf = s_ascal + 192;
    float* s_colf = s_ascal + 256;
    float* s_eref = s_ascal + 320;   // [128] 2^ref
    float* s_gC = s_ascal + 448;     // [128] g_{n-1}
    float* s_fS = s_ascal + 576;     // [128] 2^(l_{n-1} - ref)
    uint64_t* bar_v = reinterpret_cast<uint64_t*>(sm + G_OFF_SMALL + 2816);
    uint64_t* bar_mma = bar_v + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + G_OFF_SMALL + 2832);
    const uint32_t sbase = smem_u32(sm);
    auto bits_to_f32 = [](unsigned short u) { return __uint_as_float((uint32_t)u << 16); };

    // The CTA launched about `prefetch_ahead` CTAs later (the block scheduler
    // hands out CTAs in linear order as earlier ones finish) reads its q, k,
    // v and channel gates with plain loads right at its start: pull its rows
    // into L2 now, so its build waits on L2 rather than HBM latency.
    if (pp.prefetch_ahead > 0) {
        const long long lin = (long long)blockIdx.x + (long long)gridDim.x * (blockIdx.y + (long long)gridDim.y * blockIdx.z) +
                              pp.prefetch_ahead;
        const long long tot = (long long)gridDim.x * gridDim.y * gridDim.z;
        if (lin < tot) {
            const int nx = (int)(lin % gridDim.x);
            const long long yz = lin / gridDim.x;
            const int ny = (int)(yz % gridDim.y), nz = (int)(yz / gridDim.y);
            const int r = tid & 63, t = (pp.c_begin + nx) * C + r;
            if (t < T) {
                const size_t tok = (size_t)nz * T + t;
                const int part = tid >> 6;
                const char* row = nullptr;
                int bytes = 0;
                if (part == 0) { row = (const char*)(pp.q + (tok * (H / pp.group) + ny / pp.group) * DK); bytes = 2 * DK; }
                else if (part == 1) { row = (const char*)(pp.k + (tok * (H / pp.group) + ny / pp.group) * DK); bytes = 2 * DK; }
                else if (part == 2) { row = (const char*)(pp.v + (tok * H + ny) * dv); bytes = 2 * dv; }
                else if (ACH) { row = (const char*)(pp.alpha + (tok * H + ny) * DK); bytes = 2 * DK; }
                for (int off = 0; row && off < bytes; off += 128) prefetch_l2(row + off);
                if (part < 2) {
                    const bool chan = part == 0 ? pp.bkind == GDR_GATE_CHANNEL : pp.wkind == GDR_GATE_CHANNEL;
                    const __nv_bfloat16* g = part == 0 ? pp.bg : pp.wg;
                    if (chan && !(TIED && part == 1))
                        for (int off = 0; off < 2 * DK; off += 128)
                            prefetch_l2((const char*)(g + (tok * H + ny) * DK) + off);
                }
            }
        }
    }
    GDR_TRACE_G(0);
    if (tid == 0) {
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) tmem_alloc(s_tmem, G_TM_COLS);
    if (tid < C) {
        const bool valid = tid < n;
        s_ascal[tid] = (pp.akind == GDR_GATE_SCALAR && valid) ? bits_to_f32(g_a) : 1.f;
        s_bscal[tid] = (pp.bkind == GDR_GATE_SCALAR && valid) ? bits_to_f32(g_b) : 0.f;
        s_wscal[tid] = (pp.wkind == GDR_GATE_SCALAR && valid) ? bits_to_f32(g_w)
                       : (pp.wkind == GDR_GATE_NONE ? 1.f : 0.f);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t ph_v = 0, ph_mma = 0;
    bool ok = true;
    GDR_TRACE_G(1);

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

    // ---- build ------------------------------------------------------------------
    {
        float* scan = reinterpret_cast<float*>(sm + G_OFF_SCR);  // [8 rg][128 ch] + [128]
        float lrow0[4];   // channel decay: l at this thread's first token - ref
        bool out_of_range;  // the chunk's decay span exceeds the factorisation's range
        if (!ACH) {
            if (warp == 0) {
                const int lane = tid;
                const float la0 = (2 * lane < n) ? lg2_approx(s_ascal[2 * lane]) : 0.f;
                const float la1 = (2 * lane + 1 < n) ? lg2_approx(s_ascal[2 * lane + 1]) : 0.f;
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
            out_of_range = scan[3] != 0.f;
            if (tid < 128) {
                s_eref[tid] = scan[0];
                s_gC[tid] = scan[1];
                s_fS[tid] = scan[2];
            }
            __syncthreads();
        } else {
            float loc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = rg * 8 + i;
                float av[4];
                unpack4(aa[i], av);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    loc[e] += r < n ? lg2_approx(av[e]) : 0.f;  // padding tokens do not decay
                    if (i == 0) lrow0[e] = loc[e];
                }
            }
            *reinterpret_cast<float4*>(scan + rg * 128 + ch0) = make_float4(loc[0], loc[1], loc[2], loc[3]);
            if (rg == 0)
                *reinterpret_cast<float4*>(scan + 1024 + ch0) = make_float4(lrow0[0], lrow0[1], lrow0[2], lrow0[3]);
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
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float ref = 0.5f * (l0[e] + tot[e]);  // tot = l_{n-1} (padding adds 0)
                bad |= (l0[e] - tot[e]) > 230.f;
                lrow0[e] += pre[e] - ref;
                if (rg == 0) {
                    s_eref[ch0 + e] = ex2_approx(ref);
                    s_gC[ch0 + e] = ex2_approx(tot[e]);
                    s_fS[ch0 + e] = ex2_approx(tot[e] - ref);
                }
            }
            // every channel's eref / fS is needed below
            out_of_range = __syncthreads_or(bad) != 0;
        }
        if (out_of_range && tid == 0) flag_status(pp.d_status, GDR_DEVICE_DECAY_RANGE);
        GDR_TRACE_G(2);
        float er[4], fs[4];
        {
            const float4 e4 = *reinterpret_cast<const float4*>(s_eref + ch0);
            const float4 f4 = *reinterpret_cast<const float4*>(s_fS + ch0);
            er[0] = e4.x; er[1] = e4.y; er[2] = e4.z; er[3] = e4.w;
            fs[0] = f4.x; fs[1] = f4.y; fs[2] = f4.z; fs[3] = f4.w;
        }
        if (rg == 0) {
            // a negative g_{n-1} in every channel sends the chunk down the state
            // pass's exact path (this pass's other outputs for it are then unused)
            const float4 g4 = out_of_range ? make_float4(-1.f, -1.f, -1.f, -1.f)
                                           : *reinterpret_cast<const float4*>(s_gC + ch0);
            *reinterpret_cast<float4*>(pp.gc + (((size_t)bb * H + h) * nchunks + ci) * DK + ch0) = g4;
        }
        float rowf_c[4];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            {
                const int sl = i & 3;
                const int r = rg * 8 + i;
                const bool valid = r < n;
                float k4[4], q4[4], b4[4], w4[4];
                unpack4(ka[sl], k4);
                unpack4(qa[sl], q4);
                if (bch) unpack4(ba[sl], b4);
                else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) b4[e] = s_bscal[r];
                }
                if (!TIED) {
                    if (pp.wkind == GDR_GATE_TIED) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) w4[e] = b4[e];
                    } else if (wch) {
                        unpack4(wa[sl], w4);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) w4[e] = s_wscal[r];
                    }
                }
                if (i < 4) load_token(i + 4);
                if (ACH) {
                    // rowf by a multiply chain over the thread's 8 tokens (one exp2)
                    float av[4];
                    unpack4(aa[i], av);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        rowf_c[e] = (i == 0) ? ex2_approx(lrow0[e]) : rowf_c[e] * (valid ? av[e] : 1.f);
                }
                const float rs = ACH ? 0.f : s_rowf[r], cs = ACH ? 0.f : s_colf[r];
                float kb[4], qs[4], ks[4], kws[4], qg[4], k2[4], kw2[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float rowf = ACH ? rowf_c[e] : rs;
                    const float colf = ACH ? rcp_newton(rowf) : cs;
                    const float kk = valid ? k4[e] : 0.f;
                    const float qq = valid ? q4[e] : 0.f;
                    kb[e] = b4[e] * kk * rowf;
                    qs[e] = qq * rowf;
                    ks[e] = kk * colf;
                    kws[e] = TIED ? 0.f : w4[e] * kk * colf;
                    qg[e] = qs[e] * er[e];
                    k2[e] = ks[e] * fs[e];
                    kw2[e] = kws[e] * fs[e];
                }
                st4(sm + G_OFF_ROP, piece4(r, cg, 128), kb);
                st4(sm + G_OFF_ROP, piece4(64 + r, cg, 128), qs);
                st4(sm + G_OFF_COP, piece4(r, cg, N1), ks);
                if (!TIED) st4(sm + G_OFF_COP, piece4(64 + r, cg, N1), kws);
                if (valid) {
                    const size_t e = (((size_t)bb * T + t0 + r) * H + h) * DK + ch0;
                    st8b(pp.qg + e, qg);
                    st8b(pp.k2 + e, k2);
                    if (!TIED) st8b(pp.kw2 + e, kw2);
                }
            }
        }
    }
    GDR_BEFORE_MMA();
    GDR_TRACE_G(3);

    // ---- P1: D1 = [Kb ; Qs] x [Ks ; Kws]^T ---------------------------------------
    if (tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, N1, 0, 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t koff = (ks >> 2) * 16384u + (ks & 3) * 32u;
            const uint32_t koffb = (ks >> 2) * (uint32_t)(N1 * 128) + (ks & 3) * 32u;
            mma_bf16(tmem, sdesc_sw128(sbase + G_OFF_ROP + koff, 16, 1024),
                     sdesc_sw128(sbase + G_OFF_COP + koffb, 16, 1024), id, ks > 0);
        }
        mma_commit(bar_mma);
    }
    GDR_WAIT(bar_mma, ph_mma);
    tc_fence_after();
    GDR_TRACE_G(4);
    // the Qs rows are consumed: V's tiles go there (column block vt, rows 64..127)
    if (tid == 0) {
        mbar_expect_tx(bar_v, (uint32_t)nvt * 8192u);
        for (int vt = 0; vt < nvt; ++vt)
            tma_load_4d(sm + G_OFF_ROP + vt * 16384 + 8192, &tm_v, bar_v, vt * 64, h, t0, bb);
    }

    // ---- unload D1: A (fp32) + transposed diagonal blocks; Bm -> X;
    //      Aq (Bq) -> staging in L (APRE) -> workspace by bulk tensor store ----------
    {
        const int r = row & 63;
        float d[32], d2[32];
        tmem_ld32_async(tmem + lane_base + wg * 32, d);
        if (!TIED) tmem_ld32_async(tmem + lane_base + 64 + wg * 32, d2);
        tmem_wait_ld();
        if (row < 64) {
            float* A32 = reinterpret_cast<float*>(sm + G_OFF_A32);
#pragma unroll
            for (int j4 = 0; j4 < 32; j4 += 4) {
                const int j = wg * 32 + j4;
                const float4 x = make_float4(j < r ? d[j4] : 0.f, j + 1 < r ? d[j4 + 1] : 0.f,
                                             j + 2 < r ? d[j4 + 2] : 0.f, j + 3 < r ? d[j4 + 3] : 0.f);
                *reinterpret_cast<float4*>(f32_at(A32, r, j)) = x;
            }
            const int I = r >> 4, rr = r & 15;
            if ((I >> 1) == wg) {
                float* at = reinterpret_cast<float*>(sm + G_OFF_SCR) + I * 272;
                if (I & 1) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) at[j * 16 + rr] = j < rr ? d[16 + j] : 0.f;
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) at[j * 16 + rr] = j < rr ? d[j] : 0.f;
                }
            }
            if (!TIED) {
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = (wg * 32 + c8 * 8 + e < r) ? d2[c8 * 8 + e] : 0.f;
                    st_chunk(sm + G_OFF_X, sw128_chunk(r, wg * 4 + c8, 64), x);
                }
            }
        } else {
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                float x[8], y[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const bool keep = wg * 32 + c8 * 8 + e <= r;
                    x[e] = keep ? d[c8 * 8 + e] : 0.f;
                    y[e] = keep && !TIED ? d2[c8 * 8 + e] : 0.f;
                }
                st_chunk(sm + G_OFF_L, sw128_chunk(r, wg * 4 + c8, 64), x);
                if (!TIED) st_chunk(sm + G_OFF_APRE, sw128_chunk(r, wg * 4 + c8, 64), y);
            }
        }
    }
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
        tma_store_4d(&tm_aq, sm + G_OFF_L, 0, h, t0, bb);
        if (!TIED) tma_store_4d(&tm_bq, sm + G_OFF_APRE, 0, h, t0, bb);
        bulk_commit_group();
    }
    GDR_TRACE_G(5);

    // ---- T = (I + A)^-1; L = T (bf16); tied: APRE = T Diag(beta) ------------------
    {
        float* A32 = reinterpret_cast<float*>(sm + G_OFF_A32);
        float* T32 = reinterpret_cast<float*>(sm + G_OFF_T32);
        solve_unit_lower(A32, T32, reinterpret_cast<float*>(sm + G_OFF_SCR), tid, warp);
        // the Aq / Bq stores have read their staging tiles before L, APRE are rewritten
        if (tid == 0) bulk_wait_group_read0();
        __syncthreads();
        GDR_TRACE_G(6);
        const int r = tid & 63, q4 = tid >> 6;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int c8 = q4 * 2 + cc;
            float x[8];
#pragma unroll
            for (int e4 = 0; e4 < 8; e4 += 4) {
                const int j = c8 * 8 + e4;
                // the block T[0:32, 32:64] is never written by the solve: it is zero
                const float4 t4 = (j < 32 || r >= 32) ? *reinterpret_cast<const float4*>(f32_at(T32, r, j))
                                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                x[e4] = t4.x; x[e4 + 1] = t4.y; x[e4 + 2] = t4.z; x[e4 + 3] = t4.w;
            }
            st_chunk(sm + G_OFF_L, sw128_chunk(r, c8, 64), x);
            if (TIED) {
                const float4 b0 = *reinterpret_cast<const float4*>(s_bscal + c8 * 8);
                const float4 b1 = *reinterpret_cast<const float4*>(s_bscal + c8 * 8 + 4);
                x[0] *= b0.x; x[1] *= b0.y; x[2] *= b0.z; x[3] *= b0.w;
                x[4] *= b1.x; x[5] *= b1.y; x[6] *= b1.z; x[7] *= b1.w;
                st_chunk(sm + G_OFF_APRE, sw128_chunk(r, c8, 64), x);
            }
        }
    }
    GDR_BEFORE_MMA();
    GDR_TRACE_G(7);
    GDR_WAIT(bar_v, ph_v);  // V arrived during the solve
    GDR_TRACE_G(8);

    // ---- P2: D2 = T Kb (cols 0..127);  tied: D3 = T Diag(beta) V (cols 128..);
    //      general: T Bm (cols 128..191) ----------------------------------------------
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idW = idesc_bf16(128, 128, 0, 1);
        const uint32_t idP = idesc_bf16(128, dv, 0, 1);
        const uint32_t id64 = idesc_bf16(128, 64, 0, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ad = sdesc_sw128(sbase + G_OFF_L + ks * 32u, 16, 1024);
            mma_bf16(tmem, ad, sdesc_sw128(sbase + G_OFF_ROP + ks * 2048u, 16384, 1024), idW, ks > 0);
            if (TIED)
                mma_bf16(tmem + 128, sdesc_sw128(sbase + G_OFF_APRE + ks * 32u, 16, 1024),
                         sdesc_sw128(sbase + G_OFF_ROP + 8192 + ks * 2048u, 16384, 1024), idP, ks > 0);
            else
                mma_bf16(tmem + 128, ad, sdesc_sw128(sbase + G_OFF_X + ks * 2048u, 8192, 1024), id64, ks > 0);
        }
        mma_commit(bar_mma);
    }
    GDR_WAIT(bar_mma, ph_mma);
    tc_fence_after();
    GDR_TRACE_G(9);

    // ---- WN = -W 2^ref -> staging (A32 region); tied: P -> staging (T32 region);
    //      general: -T Bm -> APRE ------------------------------------------------------
    if (row < 64) {
        const int r = row;
        float d[32], d1[32];
        tmem_ld32_async(tmem + lane_base + wg * 64, d);
        tmem_ld32_async(tmem + lane_base + wg * 64 + 32, d1);
        tmem_wait_ld();
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
            float x[8];
            const float* dd = c8 < 4 ? d + c8 * 8 : d1 + (c8 - 4) * 8;
            const float4 e0 = *reinterpret_cast<const float4*>(s_eref + wg * 64 + c8 * 8);
            const float4 e1 = *reinterpret_cast<const float4*>(s_eref + wg * 64 + c8 * 8 + 4);
            x[0] = -dd[0] * e0.x; x[1] = -dd[1] * e0.y; x[2] = -dd[2] * e0.z; x[3] = -dd[3] * e0.w;
            x[4] = -dd[4] * e1.x; x[5] = -dd[5] * e1.y; x[6] = -dd[6] * e1.z; x[7] = -dd[7] * e1.w;
            st_chunk(sm + G_OFF_A32, sw128_chunk(r, wg * 8 + c8, 64), x);
        }
        if (TIED) {
            const int half = dv >> 1;
            tmem_ld32_async(tmem + lane_base + 128 + wg * half, d);
            if (half == 64) tmem_ld32_async(tmem + lane_base + 128 + wg * half + 32, d1);
            tmem_wait_ld();
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                if (c8 * 8 >= half) break;
                const float* dd = c8 < 4 ? d + c8 * 8 : d1 + (c8 - 4) * 8;
                st_chunk(sm + G_OFF_T32, sw128_chunk(r, (wg * half) / 8 + c8, 64), dd);
            }
        } else {
            tmem_ld32(tmem + lane_base + 128 + wg * 32, d);
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = -d[c8 * 8 + e];
                st_chunk(sm + G_OFF_APRE, sw128_chunk(r, wg * 4 + c8, 64), x);
            }
        }
    }
    GDR_BEFORE_MMA();
    if (tid == 0) {
        tma_store_4d(&tm_wn, sm + G_OFF_A32, 0, h, t0, bb);
        tma_store_4d(&tm_wn, sm + G_OFF_A32 + 8192, 64, h, t0, bb);
        if (TIED)
            for (int vt = 0; vt < nvt; ++vt) tma_store_4d(&tm_p, sm + G_OFF_T32 + vt * 8192, vt * 64, h, t0, bb);
        bulk_commit_group();
    }
    GDR_TRACE_G(10);
    if (!TIED) {
        // ---- P3: D3 = (-T Bm) V -> P --------------------------------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idP = idesc_bf16(128, dv, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem, sdesc_sw128(sbase + G_OFF_APRE + ks * 32u, 16, 1024),
                         sdesc_sw128(sbase + G_OFF_ROP + 8192 + ks * 2048u, 16384, 1024), idP, ks > 0);
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        if (row < 64) {
            const int r = row;
            const int half = dv >> 1;
            float d[32], d1[32];
            tmem_ld32_async(tmem + lane_base + wg * half, d);
            if (half == 64) tmem_ld32_async(tmem + lane_base + wg * half + 32, d1);
            tmem_wait_ld();
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                if (c8 * 8 >= half) break;
                const float* dd = c8 < 4 ? d + c8 * 8 : d1 + (c8 - 4) * 8;
                st_chunk(sm + G_OFF_T32, sw128_chunk(r, (wg * half) / 8 + c8, 64), dd);
            }
        }
        fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
            for (int vt = 0; vt < nvt; ++vt) tma_store_4d(&tm_p, sm + G_OFF_T32 + vt * 8192, vt * 64, h, t0, bb);
            bulk_commit_group();
        }
    }
    GDR_TRACE_G(11);

finish:
    if (!ok && tid == 0) flag_status(pp.d_status, GDR_DEVICE_TIMEOUT);
    if (tid == 0) bulk_wait_group0();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, G_TM_COLS);
#undef GDR_WAIT
#undef GDR_BEFORE_MMA
}

// ---- pass 2 ------------------------------------------------------------------
template <bool UNTIED>
struct StateLayout {
    // inputs are triple-buffered with tied gates (chunk ci + 2 loads while chunk
    // ci runs), double-buffered with independent gates (more inputs per chunk)
    static constexpr int NBUF = UNTIED ? 2 : 3;
    static constexpr uint32_t QW = 0;                          // [QG ; WN] bf16 [128 x 128], 32 KB each
    static constexpr uint32_t K2 = QW + NBUF * 32768;          // K2 bf16 [64 x 128], 16 KB each
    static constexpr uint32_t P = K2 + NBUF * 16384;           // P slice bf16 [64 x 64], 8 KB each
    static constexpr uint32_t AQ = P + NBUF * 8192;            // AQ bf16 [64 x 64], 8 KB each: rows
                                                               // 0..63 of an M = 128 operand whose
                                                               // rows 64..127 (the 8 KB after) are unused
    static constexpr uint32_t KW2 = AQ + NBUF * 8192;          // KW2 bf16 [64 x 128], 16 KB each (untied)
    static constexpr uint32_t BQ = KW2 + (UNTIED ? NBUF * 16384 : 0);  // BQ bf16 [64 x 64] (untied)
    static constexpr uint32_t V = BQ + (UNTIED ? NBUF * 8192 : 0);     // V slice bf16 [64 x 64] (untied)
    static constexpr uint32_t U = V + (UNTIED ? NBUF * 8192 : 0);      // U bf16 [64 x 64]
    static constexpr uint32_t SBF = U + 8192;                          // S bf16 [128 x 64]
    static constexpr uint32_t EXR = SBF + 16384;                       // exact-path scratch (2.5 KB)
    static constexpr uint32_t SMALL = EXR + 2560;                      // barriers, TMEM slot (1 KB)
    static constexpr uint32_t BYTES = SMALL + 1024 + 1024;
};
// D3 ([QG S ; U - P]) and D5 (AQ U (+ BQ V), lanes 0..63) alternate between two
// column sets; D4 = K2^T U (+ KW2^T V).
constexpr uint32_t GS_TM_D3 = 0, GS_TM_D5 = 128, GS_TM_D4 = 256, GS_TM_COLS = 512;
constexpr int GS_NT = 288;  // warps 0..7 compute, warp 8 issues MMAs and TMA loads

struct GStateParams {
    const float* S0;  // state at chunk c_begin (NULL: zero)
    const float* gc;  // g_{n-1} per chunk and channel; negative: take the exact path
    ExactArgs ex;     // raw inputs for chunks that take the exact path
    int group;        // value heads per q/k head
    __nv_bfloat16* o;
    float* ST;        // state after chunk c_end - 1 (NULL: not written); may alias S0
    int* d_status;
    int T, H, dv;
    int c_begin, c_end;  // chunk range of this launch
};

__device__ __forceinline__ bool gs_compute_bar_and(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.and.pred q, 1, 256, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void gs_mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Chunk step. The chain from one chunk to the next holds only the products
// that depend on the state:
//   D3 = [QG ; WN] S          (U = P + WN S in lanes 64..127, by warps 2, 3, 6, 7)
//   D4 = K2^T U (+ KW2^T V)   (S <- Diag(g_{n-1}) S + D4, warps 0..7)
// and after it, from the same issuing warp (warp 8), D5 = [AQ ; .] U (+ [BQ ; .]
// V); O = QG S + AQ U (+ BQ V), lanes 0..63, is written by warps 0, 1, 4, 5
// during the next chunk. No product is in flight while U is written: their
// operand reads would take the shared-memory bandwidth the unload needs. A chunk marked by the first pass
// (negative g_{n-1}: its decay span does not fit two bounded factors) is
// applied token by token from the raw inputs instead, with no MMA.
template <bool UNTIED>
__global__ void __launch_bounds__(GS_NT, 1) state_general_kernel(
    const __grid_constant__ CUtensorMap tm_wn, const __grid_constant__ CUtensorMap tm_qg,
    const __grid_constant__ CUtensorMap tm_k2, const __grid_constant__ CUtensorMap tm_aq,
    const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_kw2,
    const __grid_constant__ CUtensorMap tm_bq, const __grid_constant__ CUtensorMap tm_v,
    const GStateParams p) {
    using Lay = StateLayout<UNTIED>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = (warp >> 2) & 1, row = tid & 127;
    const bool lo = row < 64;
    const int vt = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int v0 = vt * NV;
    const int T = p.T, H = p.H;
    const int nchunks = (T + C - 1) / C;

    constexpr int NBUF = Lay::NBUF;
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + Lay::SMALL);  // [3]
    uint64_t* bar_w = bar_tma + 3;
    uint64_t* bar_k = bar_tma + 4;
    uint64_t* bar_a = bar_tma + 5;
    uint64_t* bar_drain = bar_tma + 6;
    uint64_t* u_ready = bar_tma + 7;
    uint64_t* s_ready = bar_tma + 8;
    // D5 commits, one barrier per TMEM column set (chunk parity): a barrier completes
    // every second chunk, so a wait for one chunk's completion can never see the next
    // completion of the same barrier first (that needs the state step in between)
    auto bar_a_set = [&](int set) { return bar_tma + 5 + 4 * set; };  // bar_a, bar_tma + 9
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + Lay::SMALL + 128);
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bar_tma[i], 1);
        mbar_init(bar_w, 1);
        mbar_init(bar_k, 1);
        mbar_init(bar_a, 1);
        mbar_init(bar_drain, 1);
        mbar_init(u_ready, 128);
        mbar_init(s_ready, 1);
        mbar_init(bar_a_set(1), 1);
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(s_tmem, GS_TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    bool ok = true;
    const uint32_t sbase = smem_u32(sm);
    const int c_begin = p.c_begin, c_end = p.c_end;
    const float* gch = p.gc + ((size_t)bb * H + h) * nchunks * DK;  // [nchunks][128]

    auto issue_loads = [&](int ci) {
        const int t0 = ci * C, buf = ci % NBUF;
        uint64_t* bar = &bar_tma[buf];
        uint8_t* qw = sm + Lay::QW + buf * 32768;
        mbar_expect_tx(bar, (UNTIED ? 12u : 8u) * 8192u);
        // [QG ; WN]: each 64-column block holds 128 rows (QG rows 0..63, WN rows 64..127)
        tma_load_4d(qw, &tm_qg, bar, 0, h, t0, bb);
        tma_load_4d(qw + 16384, &tm_qg, bar, 64, h, t0, bb);
        tma_load_4d(qw + 8192, &tm_wn, bar, 0, h, t0, bb);
        tma_load_4d(qw + 16384 + 8192, &tm_wn, bar, 64, h, t0, bb);
        tma_load_4d(sm + Lay::K2 + buf * 16384, &tm_k2, bar, 0, h, t0, bb);
        tma_load_4d(sm + Lay::K2 + buf * 16384 + 8192, &tm_k2, bar, 64, h, t0, bb);
        tma_load_4d(sm + Lay::AQ + buf * 8192, &tm_aq, bar, 0, h, t0, bb);
        tma_load_4d(sm + Lay::P + buf * 8192, &tm_p, bar, v0, h, t0, bb);
        if (UNTIED) {
            tma_load_4d(sm + Lay::KW2 + buf * 16384, &tm_kw2, bar, 0, h, t0, bb);
            tma_load_4d(sm + Lay::KW2 + buf * 16384 + 8192, &tm_kw2, bar, 64, h, t0, bb);
            tma_load_4d(sm + Lay::BQ + buf * 8192, &tm_bq, bar, 0, h, t0, bb);
            tma_load_4d(sm + Lay::V + buf * 8192, &tm_v, bar, v0, h, t0, bb);
        }
    };

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
        for (int ch = 0; ch < 4; ++ch) st_chunk(sm + Lay::SBF, sw128_chunk(row, wg * 4 + ch, DK), &S[8 * ch]);
    }
    // the state's bf16 copy is read by the first MMA batch (async proxy)
    fence_proxy_async();
    tc_fence_before();
    if (warp == 8 && lane == 0)
        for (int ci = c_begin; ci < c_end && ci < c_begin + NBUF - 1; ++ci) issue_loads(ci);
    __syncthreads();

    if (warp == 8) {
        // ---------------- issuer warp ------------------------------------------------
        bool iok = true;
        int nm = 0;            // chunks taken on the tensor cores so far
        int loads_issued = min(c_end, c_begin + NBUF - 1);
        bool prev_mma = false;  // chunk ci - 1 ran on the tensor cores (its AQ U may be in flight)
        for (int ci = c_begin; ci < c_end; ++ci) {
            const int buf = ci % NBUF, par = nm & 1;
            const uint32_t qwb = sbase + Lay::QW + buf * 32768u;
            const uint32_t k2b = sbase + Lay::K2 + buf * 16384u;
            const uint32_t aqa = sbase + Lay::AQ + buf * 8192u;  // AQ = rows 0..63
            const uint32_t ub = sbase + Lay::U;
            const uint32_t d3 = GS_TM_D3 + (uint32_t)par * 64u, d5 = GS_TM_D5 + (uint32_t)par * 64u;
            const bool exact = gch[(size_t)ci * DK] < 0.f;
            iok = mbar_wait(&bar_tma[buf], (uint32_t)(((ci - c_begin) / NBUF) & 1)) && iok;
            if (ci > c_begin) iok = mbar_wait(s_ready, (uint32_t)((ci - 1 - c_begin) & 1)) && iok;
            // the stage of chunk ci - 1 is refilled below: its AQ tile's last reader done
            if (prev_mma) iok = mbar_wait(bar_a_set((nm - 1) & 1), (uint32_t)(((nm - 1) >> 1) & 1)) && iok;
            iok = __all_sync(0xffffffffu, iok);
            if (!iok) break;
            tc_fence_after();
            if (lane == 0) {
                if (!exact) {
                    const uint32_t idS = idesc_bf16(128, NV, 0, 1);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t koff = (ks >> 2) * 16384u + (ks & 3) * 32u;
                        mma_bf16(tmem + d3, sdesc_sw128(qwb + koff, 16, 1024),
                                 sdesc_sw128(sbase + Lay::SBF + ks * 2048u, 8192, 1024), idS, ks > 0);
                    }
                    mma_commit(bar_w);
                }
                // chunk ci + NBUF - 1's inputs go to the buffers of chunk ci - 1
                if (ci + NBUF - 1 < c_end) issue_loads(ci + NBUF - 1);
            }
            if (ci + NBUF - 1 < c_end) loads_issued = ci + NBUF;
            __syncwarp();
            if (!exact) {
                iok = __all_sync(0xffffffffu, mbar_wait(u_ready, (uint32_t)(nm & 1)) && iok);
                if (!iok) break;
                tc_fence_after();
                if (lane == 0) {
                    // ---- D4 = K2^T U (+ KW2^T V), then D5 = [AQ ; .] U (+ [BQ ; .] V): the
                    //      products with V come after the state's, and no product runs
                    //      while U is being written (its shared-memory reads would slow it)
                    const uint32_t idM = idesc_bf16(128, NV, 1, 1);
                    const uint32_t vb = sbase + Lay::V + buf * 8192u;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16(tmem + GS_TM_D4, sdesc_sw128(k2b + ks * 2048u, 8192, 1024),
                                 sdesc_sw128(ub + ks * 2048u, 8192, 1024), idM, ks > 0);
                    if (UNTIED)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_bf16(tmem + GS_TM_D4, sdesc_sw128(sbase + Lay::KW2 + buf * 16384u + ks * 2048u, 8192, 1024),
                                     sdesc_sw128(vb + ks * 2048u, 8192, 1024), idM, 1u);
                    mma_commit(bar_k);
                    const uint32_t idK = idesc_bf16(128, NV, 0, 1);
                    const uint32_t bqa = sbase + Lay::BQ + buf * 8192u;  // BQ = rows 0..63
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16(tmem + d5, sdesc_sw128(aqa + ks * 32u, 16, 1024),
                                 sdesc_sw128(ub + ks * 2048u, 8192, 1024), idK, ks > 0);
                    if (UNTIED)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_bf16(tmem + d5, sdesc_sw128(bqa + ks * 32u, 16, 1024),
                                     sdesc_sw128(vb + ks * 2048u, 8192, 1024), idK, 1u);
                    mma_commit(bar_a_set(par));
                }
                __syncwarp();
                ++nm;
            }
            prev_mma = !exact;
        }
        if (!iok) {
            ok = false;
            if (lane == 0) {
                // before the block leaves (each wait bounded): the requested input
                // copies have landed and the issued MMAs have finished
                for (int ci = max(c_begin, loads_issued - NBUF); ci < loads_issued; ++ci)
                    (void)mbar_wait(&bar_tma[ci % NBUF], (uint32_t)(((ci - c_begin) / NBUF) & 1));
                mma_commit(bar_drain);
                (void)mbar_wait(bar_drain, 0);
            }
            __syncwarp();
        }
    } else {
        // ---------------- compute warps ------------------------------------------------
        const float* gcp = gch + row;
        float gC_next = c_begin < c_end ? gcp[(size_t)c_begin * DK] : 0.f;
        auto store_o = [&](int cj, int pj) {
            const int t = cj * C + row;
            float d[32], d5[32];
            tmem_ld32_async(tmem + lane_base + GS_TM_D3 + pj * 64 + wg * 32, d);
            tmem_ld32_async(tmem + lane_base + GS_TM_D5 + pj * 64 + wg * 32, d5);
            tmem_wait_ld();
            if (t < T) {
#pragma unroll
                for (int j = 0; j < 32; ++j) d[j] += d5[j];
                st32_bf16(p.o + (((size_t)bb * T + t) * H + h) * p.dv + v0 + wg * 32, d, 1.f);
            }
        };
        bool w_ok = true;
        int nm = 0;
        int pend = -1, pend_set = 0;  // chunk whose O still sits in TMEM
        uint32_t pend_ph = 0;
        int ci = c_begin;
        for (; ci < c_end; ++ci) {
            const int buf = ci % NBUF, par = nm & 1;
            const uint32_t ph = (uint32_t)(nm & 1);
            const uint32_t d3 = GS_TM_D3 + (uint32_t)par * 64u;
            const float gC = gC_next;
            if (ci + 1 < c_end) gC_next = gcp[(size_t)(ci + 1) * DK];
            const bool exact = gC < 0.f;  // the same mark in every channel: uniform
            if (lo && pend >= 0) {
                w_ok = mbar_wait(bar_a_set(pend_set), pend_ph) && w_ok;
                tc_fence_after();
                store_o(pend, pend_set);
            }
            pend = -1;
            if (exact) {
                exact_tokens(p.ex, S, reinterpret_cast<float*>(sm + Lay::EXR), bb, h, h / p.group, v0,
                             ci * C, min(C, T - ci * C), tid);
            } else {
                if (!lo) {
                    // ---- U = P + WN S (lanes 64..127 of D3) -> U --------------------------
                    w_ok = mbar_wait(&bar_tma[buf], (uint32_t)(((ci - c_begin) / NBUF) & 1)) && w_ok;
                    w_ok = mbar_wait(bar_w, ph) && w_ok;
                    tc_fence_after();
                    {
                        const int j = row - 64;
                        float d[32];
                        tmem_ld32(tmem + lane_base + d3 + wg * 32, d);
#pragma unroll
                        for (int c8 = 0; c8 < 4; ++c8) {
                            float x[8];
                            const uint32_t off = sw128_chunk(j, wg * 4 + c8, 64);
                            ld_chunk(sm + Lay::P + buf * 8192, off, x);
#pragma unroll
                            for (int e = 0; e < 8; ++e) x[e] += d[c8 * 8 + e];
                            st_chunk(sm + Lay::U, off, x);
                        }
                    }
                    fence_proxy_async();
                    tc_fence_before();
                    gs_mbar_arrive(u_ready);
                }
                // ---- S = Diag(GC) S + D4 -------------------------------------------------
                w_ok = mbar_wait(bar_k, ph) && w_ok;
                tc_fence_after();
                {
                    float dS[32];
                    tmem_ld32(tmem + lane_base + GS_TM_D4 + wg * 32, dS);
#pragma unroll
                    for (int j = 0; j < NH; ++j) S[j] = fmaf(gC, S[j], dS[j]);
                }
                pend = ci;
                pend_set = par;
                pend_ph = (uint32_t)((nm >> 1) & 1);  // the set's own completion count
                ++nm;
            }
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) st_chunk(sm + Lay::SBF, sw128_chunk(row, wg * 4 + ch, DK), &S[8 * ch]);
            fence_proxy_async();  // the state copy feeds the next chunk's MMAs
            tc_fence_before();
            if (!gs_compute_bar_and(w_ok)) break;
            if (tid == 0) gs_mbar_arrive(s_ready);
        }
        if (ci < c_end) ok = false;  // a wait gave up
        if (ok && lo && pend >= 0) {
            ok = mbar_wait(bar_a_set(pend_set), pend_ph);
            tc_fence_after();
            if (ok) store_o(pend, pend_set);
        }
        if (!gs_compute_bar_and(ok)) ok = false;
        if (ok && p.ST) {
            float* st = p.ST + (((size_t)bb * H + h) * DK + row) * p.dv + v0 + wg * NH;
#pragma unroll
            for (int j = 0; j < NH; j += 4) *reinterpret_cast<float4*>(st + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }
    if (!ok && (tid == 0 || tid == 256)) flag_status(p.d_status, GDR_DEVICE_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, GS_TM_COLS);
}

}  // namespace twopass_g

// Workspace of the general two-pass path: sub-buffers in this order, each
// rounded up to 256 bytes: WN, QG, K2, AQ, P, [KW2, BQ], GC, and the fp32
// state carried between the segments of a segmented state pass.
struct GeneralWorkspace {
    size_t off[9];
    size_t total;
};

static GeneralWorkspace general_workspace_layout(int B, int T, int H, int dv, bool untied) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t tok = (size_t)B * T * H;
    const size_t nchunks = ((size_t)T + 63) / 64;
    const size_t sizes[9] = {tok * 128 * 2, tok * 128 * 2, tok * 128 * 2, tok * 64 * 2,
                             tok * (size_t)dv * 2, untied ? tok * 128 * 2 : 0, untied ? tok * 64 * 2 : 0,
                             (size_t)B * H * nchunks * 128 * 4, (size_t)B * H * 128 * (size_t)dv * 4};
    GeneralWorkspace w;
    size_t o = 0;
    for (int i = 0; i < 9; ++i) {
        w.off[i] = o;
        o += up(sizes[i]);
    }
    w.total = o;
    return w;
}

size_t twopass_general_workspace_bytes(int B, int T, int H, int dv, bool untied) {
    return general_workspace_layout(B, T, H, dv, untied).total;
}

using MapFn = bool (*)(CUtensorMap*, const void*, int, int, int, int);

// Segmented state pass: segments of at least kSegMin chunks, at most
// kMaxSegments. The auxiliary stream and events are created on the first
// segmented call on a device and kept for the process. They are shared by
// every call on that device, so a call holds the device's lock from its first
// event record to its last stream wait: another call's records can then never
// be the ones this call waits on. A call that finds the lock taken, or whose
// stream is being captured into a graph, does not segment (one prep launch,
// one state launch on the caller's stream).
constexpr int kSegMin = 32;
constexpr int kMaxSegments = 8;

struct AuxResources {
    std::mutex mu;  // held for a whole segmented enqueue sequence
    cudaStream_t stream = nullptr;
    cudaEvent_t events[kMaxSegments + 1] = {};
    bool ready = false;
};

static AuxResources* aux_resources(int dev) {
    static std::mutex create_mu;
    static AuxResources res[64];
    if (dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(create_mu);
    AuxResources& r = res[dev];
    if (!r.ready) {
        cudaStream_t s = nullptr;
        if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
        for (int i = 0; i <= kMaxSegments; ++i)
            if (cudaEventCreateWithFlags(&r.events[i], cudaEventDisableTiming) != cudaSuccess) {
                for (int j = 0; j < i; ++j) cudaEventDestroy(r.events[j]);
                cudaStreamDestroy(s);
                return nullptr;
            }
        r.stream = s;
        r.ready = true;
    }
    return &r;
}

// maps: q, k, v (of the call). alpha/b/w kinds as in the C ABI.
cudaError_t launch_chunk_twopass_general(const CUtensorMap* maps, MapFn make_map, void* ws,
                                         const void* q, const void* k, const void* v, const void* alpha,
                                         const void* b, const void* w, int akind, int bkind,
                                         int wkind, const float* S0, void* o, float* ST,
                                         int* d_status, int B, int T, int H, int dv, int group,
                                         bool allow_segments, cudaStream_t st) {
    using namespace twopass_g;
    const bool tied = wkind == GDR_GATE_TIED && bkind == GDR_GATE_SCALAR;
    const bool ach = akind == GDR_GATE_CHANNEL;
    const GeneralWorkspace lay = general_workspace_layout(B, T, H, dv, !tied);
    uint8_t* base = reinterpret_cast<uint8_t*>(ws);
    auto at = [&](int i) { return reinterpret_cast<__nv_bfloat16*>(base + lay.off[i]); };

    GPrepParams pp;
    pp.q = reinterpret_cast<const __nv_bfloat16*>(q);
    pp.k = reinterpret_cast<const __nv_bfloat16*>(k);
    pp.alpha = reinterpret_cast<const __nv_bfloat16*>(alpha);
    pp.bg = reinterpret_cast<const __nv_bfloat16*>(b);
    pp.wg = reinterpret_cast<const __nv_bfloat16*>(w);
    pp.wn = at(0); pp.qg = at(1); pp.k2 = at(2); pp.aq = at(3); pp.p = at(4);
    pp.kw2 = at(5); pp.bq = at(6);
    pp.gc = reinterpret_cast<float*>(base + lay.off[7]);
    pp.d_status = d_status;
    pp.T = T; pp.H = H; pp.dv = dv;
    pp.akind = akind; pp.bkind = bkind; pp.wkind = wkind;
    pp.group = group;
    pp.v = reinterpret_cast<const __nv_bfloat16*>(v);
    pp.prefetch_ahead = 0;
    CUtensorMap sm_maps[8];
    const int dims[7] = {128, 128, 128, 64, dv, 128, 64};
    for (int i = 0; i < 7; ++i) {
        const void* ptr = (i >= 5 && tied) ? base + lay.off[0] : base + lay.off[i];
        const int d = (i >= 5 && tied) ? 128 : dims[i];
        if (!make_map(&sm_maps[i], ptr, B, T, H, d)) return cudaErrorInvalidValue;
    }
    sm_maps[7] = maps[2];
    // the untied maps stand in for the tied form's unused Bq output
    const CUtensorMap& bq_map = tied ? sm_maps[3] : sm_maps[6];

    const int nchunks = (T + C - 1) / C;
    int nsm_p = 0, dev_p = 0;
    if (cudaGetDevice(&dev_p) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm_p, cudaDevAttrMultiProcessorCount, dev_p) != cudaSuccess)
        nsm_p = 0;
    // resident first-pass CTAs: two per SM, less the SMs a concurrent state pass holds
    auto prep_range = [&](int c0, int c1, cudaStream_t stream, int busy_sms) -> cudaError_t {
        GPrepParams pr = pp;
        pr.c_begin = c0;
        pr.prefetch_ahead = max(0, 2 * (nsm_p - busy_sms));
        const dim3 pgrid(c1 - c0, H, B);
        auto go = [&](auto kern) -> cudaError_t {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G_SMEM_BYTES);
            if (e != cudaSuccess) return e;
            kern<<<pgrid, NT, G_SMEM_BYTES, stream>>>(maps[2], sm_maps[0], sm_maps[3], sm_maps[4], bq_map, pr);
            return cudaGetLastError();
        };
        return tied ? (ach ? go(prep_general_kernel<true, true>) : go(prep_general_kernel<true, false>))
                    : (ach ? go(prep_general_kernel<false, true>) : go(prep_general_kernel<false, false>));
    };
    GStateParams sp;
    sp.gc = pp.gc; sp.o = reinterpret_cast<__nv_bfloat16*>(o);
    sp.ex.q = pp.q; sp.ex.k = pp.k; sp.ex.v = reinterpret_cast<const __nv_bfloat16*>(v);
    sp.ex.alpha = pp.alpha; sp.ex.b = pp.bg; sp.ex.w = pp.wg;
    sp.ex.akind = akind; sp.ex.bkind = bkind; sp.ex.wkind = wkind;
    sp.ex.o = sp.o; sp.ex.T = T; sp.ex.H = H; sp.ex.Hq = H / group; sp.ex.dv = dv;
    sp.group = group;
    sp.d_status = d_status; sp.T = T; sp.H = H; sp.dv = dv;
    const dim3 sgrid(dv / NV, H, B);
    auto state_range = [&](int c0, int c1, const float* s_in, float* s_out) -> cudaError_t {
        GStateParams sr = sp;
        sr.c_begin = c0; sr.c_end = c1; sr.S0 = s_in; sr.ST = s_out;
        auto go = [&](auto kern, uint32_t bytes) -> cudaError_t {
            cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
            if (e2 != cudaSuccess) return e2;
            kern<<<sgrid, GS_NT, bytes, st>>>(sm_maps[0], sm_maps[1], sm_maps[2], sm_maps[3], sm_maps[4],
                                           sm_maps[5], sm_maps[6], sm_maps[7], sr);
            return cudaGetLastError();
        };
        return tied ? go(state_general_kernel<false>, StateLayout<false>::BYTES)
                    : go(state_general_kernel<true>, StateLayout<true>::BYTES);
    };

    // With few state CTAs (few heads, long sequences) most SMs would idle during
    // the state pass: split the chunks into segments and let pass 1 of later
    // segments run on an auxiliary stream while the state pass works through
    // earlier ones (ordered by events only).
    int nseg = 1;
    AuxResources* aux = nullptr;
    std::unique_lock<std::mutex> aux_lock;
    int dev = 0, nsm = 0;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (allow_segments && cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        (int)(sgrid.x * sgrid.y * sgrid.z) * 2 <= nsm && nchunks >= 2 * kSegMin &&
        cudaStreamIsCapturing(st, &cap) == cudaSuccess && cap == cudaStreamCaptureStatusNone &&
        (aux = aux_resources(dev)) != nullptr) {
        aux_lock = std::unique_lock<std::mutex>(aux->mu, std::try_to_lock);
        if (aux_lock.owns_lock()) nseg = min(kMaxSegments, nchunks / kSegMin);
    }
    if (nseg == 1) {
        cudaError_t e = prep_range(0, nchunks, st, 0);
        if (e != cudaSuccess) return e;
        return state_range(0, nchunks, S0, ST);
    }
    cudaEvent_t* evs = aux->events;
    float* carry = reinterpret_cast<float*>(base + lay.off[8]);
    cudaError_t e = cudaEventRecord(evs[kMaxSegments], st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(aux->stream, evs[kMaxSegments], 0);
    for (int sgi = 0; sgi < nseg && e == cudaSuccess; ++sgi) {
        const int c0 = (int)((long long)nchunks * sgi / nseg), c1 = (int)((long long)nchunks * (sgi + 1) / nseg);
        e = prep_range(c0, c1, sgi == 0 ? st : aux->stream, sgi == 0 ? 0 : (int)(sgrid.x * sgrid.y * sgrid.z));
        if (e == cudaSuccess && sgi > 0) e = cudaEventRecord(evs[sgi], aux->stream);
    }
    for (int sgi = 0; sgi < nseg && e == cudaSuccess; ++sgi) {
        const int c0 = (int)((long long)nchunks * sgi / nseg), c1 = (int)((long long)nchunks * (sgi + 1) / nseg);
        if (sgi > 0) e = cudaStreamWaitEvent(st, evs[sgi], 0);
        if (e == cudaSuccess)
            e = state_range(c0, c1, sgi == 0 ? S0 : carry, sgi == nseg - 1 ? ST : carry);
    }
    // every wait of this call is enqueued: later records cannot affect them
    return e;
}

}  // namespace gdr

#ifdef GDR_TRACE_PHASES
extern "C" int gdr_trace_general_read(unsigned long long* host, int n) {
    return (int)cudaMemcpyFromSymbol(host, gdr::twopass_g::g_trace3, sizeof(unsigned long long) * n);
}
#endif
