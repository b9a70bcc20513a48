// Chunkwise-parallel gated delta-rule forward on sm_100a tensor cores.
//
// Math (per head, chunk of C = 64 tokens r = 0..n-1, state S at chunk start;
// "Recurrent Memory: Write, Erase, Decay, Read" sections 03-05 for the
// reassociation into chunks and the prefix sum of log decays; "Erase-then-
// Delta Attention" abstract for the chunkwise WY form with the decay absorbed
// into the erase factors):
//   l_r   = sum_{j<=r} log2 alpha_j (per channel),   g_r = 2^l_r
//   ref   = (l_0 + l_{n-1}) / 2 per channel,  rowf_r = 2^(l_r - ref),
//           colf_r = 2^(ref - l_r)  (rowf_r colf_j = g_r / g_j; both bounded)
//   Kb = b.k.rowf, Qs = q.rowf, Ks = k.colf, Kws = w.k.colf
//   A  = strict_lower(Kb Ks^T)   Bm = strict_lower(Kb Kws^T)
//   Aq = lower(Qs Ks^T)          Bq = lower(Qs Kws^T)
//   T  = (I + A)^-1                                  (unit lower triangular)
//   W  = T Kb . 2^ref            (the rows of b.k.g, mapped through T)
//   U  = -W S - T Bm V                               (per-chunk "new values")
//   O  = (Qs . 2^ref) S + Aq U + Bq V                (the chunk's outputs)
//   S' = Diag(g_{n-1}) S + Diag(2^(l_{n-1}-ref)) (Ks^T U + Kws^T V)
// With tied scalar gates b = w = beta: Bm = A Diag(beta), Bq = Aq Diag(beta),
// U + Diag(beta) V = T Diag(beta) V - W S, and only Ks^T (U + beta V) enters S'.
//
// One CTA (256 threads, two warpgroups that split every phase) owns one
// (batch, head, 64-column slice of d_v) and walks the chunks in order; its
// state slice stays on chip (fp32 registers: one row and half the columns per
// thread; a bf16 copy in shared memory as an MMA operand). Per chunk the tcgen05
// MMAs (fp32 accumulators in tensor memory) are:
//   P1  D1  = [Kb ; Qs] x [Ks ; Kws]^T                   -> A, Aq (Bm, Bq)
//   P2  D2  = [T ; 0] x [Kb | Bm]                         -> W (and T Bm)
//   P3  D3  = [T Diag(beta) ; 0] x V   or   [-T Bm ; Bq] x V    (pre-load)
//   S1  D3 += [-W ; Qs.2^ref] x S                         -> U, O partial
//   S2  D3 += [0 ; Aq] x U   and   D4 = [Ks ; Kws]^T x [U ; V]
// q, k, v and channel gates arrive by TMA (128-byte swizzle) straight into
// the operand layout the MMAs read. The unit lower triangular solve runs on
// CUDA cores in fp32 (16 x 16 diagonal blocks by forward substitution, then
// recursive halving: 16 -> 32 -> 64).
#include "chunk_common.cuh"

namespace gdr {
namespace chunk {

using namespace chunkc;

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t OFF_QIN = 0;        // q chunk [64 x 128] bf16: 2 column blocks of 8 KB
constexpr uint32_t OFF_KIN = 16384;    // k chunk
constexpr uint32_t OFF_GA = 32768;     // channel alpha chunk
constexpr uint32_t OFF_GB = 49152;     // channel b chunk
constexpr uint32_t OFF_GW = 65536;     // channel w chunk
//   reused once the operands are built:
constexpr uint32_t OFF_A32 = 0;        // A fp32 [64 x 64] (float4 groups swizzled by row)
constexpr uint32_t OFF_T32 = 16384;    // T fp32 [64 x 64]
constexpr uint32_t OFF_X = 32768;      // Bm bf16 [64 x 64] (general gates)
constexpr uint32_t OFF_P32 = 40960;    // solve scratch fp32 (8 KB): transposed diagonal blocks, then X / Y
constexpr uint32_t OFF_L = 49152;      // [T ; 0] bf16 [128 x 64]
constexpr uint32_t OFF_V = 81920;      // v slice [64 x 64] bf16, two buffers
constexpr uint32_t OFF_ROP = 98304;    // [Kb ; Qs] bf16 [128 x 128], later [-W ; Qs.2^ref]
constexpr uint32_t OFF_COP = 131072;   // [Ks ; Kws] bf16 [64 or 128 x 128]
constexpr uint32_t OFF_APRE = 163840;  // [T Diag(beta) ; 0] or [-T Bm ; Bq] bf16 [128 x 64]
constexpr uint32_t OFF_AQ = 180224;    // [0 ; Aq] bf16 [128 x 64]
constexpr uint32_t OFF_SBF = 196608;   // S bf16 [128 x 64]
constexpr uint32_t OFF_U = 212992;     // U bf16 [64 x 64]
constexpr uint32_t OFF_SCAN = 212992;  // scan scratch fp32 [9 x 128] (over U, during the build)
constexpr uint32_t OFF_SMALL = 225792; // per-token / per-channel scalars, barriers
constexpr uint32_t SMALL_BYTES = 4096;
constexpr uint32_t SMEM_BYTES = OFF_SMALL + SMALL_BYTES + 1024;  // + alignment slack

// TMEM columns
constexpr uint32_t TM_D1 = 0, TM_D2 = 128, TM_D3 = 320, TM_D4 = 384, TM_COLS = 512;

// Optional phase tracing (build with -DGDR_TRACE_PHASES): thread 0 of the
// first CTA stamps clock64() at each phase boundary of its first 64 chunks;
// gdr_trace_read() copies the stamps out. Compiled out by default.
#ifdef GDR_TRACE_PHASES
__device__ unsigned long long g_trace[64 * 16];
#define GDR_TRACE(k)                                                                          \
    do {                                                                                     \
        if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0 &&   \
            ci < 64)                                                                         \
            g_trace[ci * 16 + (k)] = clock64();                                              \
    } while (0)
#else
#define GDR_TRACE(k) \
    do {            \
    } while (0)
#endif

template <bool TIED, bool ACH>
__global__ void __launch_bounds__(NT, 1) chunk_fwd_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
    const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_w,
    const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int wg = warp >> 2;          // warpgroup: which half of the columns it handles
    const int row = tid & 127;         // TMEM lane this thread reads (warp % 4 selects the quarter)
    const int vt = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int hq = h / p.group;  // q / k head of this value head
    const int v0 = vt * NV;
    const int T = p.T, H = p.H;
    const int nchunks = (T + C - 1) / C;
    constexpr bool ach = ACH;  // channel-wise decay
    const bool bch = p.bkind == GDR_GATE_CHANNEL,
               wch = p.wkind == GDR_GATE_CHANNEL;
    constexpr int N1 = TIED ? 64 : 128;  // rows of [Ks ; Kws]

    float* s_ascal = reinterpret_cast<float*>(sm + OFF_SMALL);  // [64] scalar alpha
    float* s_bscal = s_ascal + 64;                              // [64] scalar b
    float* s_wscal = s_ascal + 128;                             // [64] scalar w
    float* s_rowf = s_ascal + 192;                              // [64] scalar-decay rowf
    float* s_colf = s_ascal + 256;                              // [64] scalar-decay colf
    float* s_eref = s_ascal + 320;                              // [128] 2^ref
    float* s_gC = s_ascal + 448;                                // [128] g_{n-1}
    float* s_fS = s_ascal + 576;                                // [128] 2^(l_{n-1}-ref)
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + OFF_SMALL + 3072);
    uint64_t* bar_mma = bar_tma + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + OFF_SMALL + 3088);

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
        const uint32_t bytes = (uint32_t)(4 + 1 + 2 * (ach + bch + wch)) * 8192u;
        mbar_expect_tx(bar_tma, bytes);
        tma_load_4d(sm + OFF_QIN, &tm_q, bar_tma, 0, hq, t0, bb);
        tma_load_4d(sm + OFF_QIN + 8192, &tm_q, bar_tma, 64, hq, t0, bb);
        tma_load_4d(sm + OFF_KIN, &tm_k, bar_tma, 0, hq, t0, bb);
        tma_load_4d(sm + OFF_KIN + 8192, &tm_k, bar_tma, 64, hq, t0, bb);
        tma_load_4d(sm + OFF_V + (ci & 1) * 8192, &tm_v, bar_tma, v0, h, t0, bb);
        if (ach) {
            tma_load_4d(sm + OFF_GA, &tm_a, bar_tma, 0, h, t0, bb);
            tma_load_4d(sm + OFF_GA + 8192, &tm_a, bar_tma, 64, h, t0, bb);
        }
        if (bch) {
            tma_load_4d(sm + OFF_GB, &tm_b, bar_tma, 0, h, t0, bb);
            tma_load_4d(sm + OFF_GB + 8192, &tm_b, bar_tma, 64, h, t0, bb);
        }
        if (wch) {
            tma_load_4d(sm + OFF_GW, &tm_w, bar_tma, 0, h, t0, bb);
            tma_load_4d(sm + OFF_GW + 8192, &tm_w, bar_tma, 64, h, t0, bb);
        }
    };

    // ---- initial state: row `row`, columns [32 wg, 32 wg + 32) of the slice ----
    constexpr int NH = NV / 2;  // state columns per thread
    float S[NH];
    {
        const float* s0 = p.S0 ? p.S0 + (((size_t)bb * H + h) * DK + row) * p.dv + v0 + wg * NH : nullptr;
#pragma unroll
        for (int j = 0; j < NH; j += 4) {
            float4 x = s0 ? *reinterpret_cast<const float4*>(s0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) st_chunk(sm + OFF_SBF, sw128_chunk(row, wg * 4 + ch, DK), &S[8 * ch]);
        if (tid < 64) {  // AQ rows 0..63 stay zero; with tied gates so do APRE rows 64..127
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                st_zero_chunk(sm + OFF_AQ, sw128_chunk(tid, ch, 128));
                if (TIED) st_zero_chunk(sm + OFF_APRE, sw128_chunk(64 + tid, ch, 128));
            }
        }
    }
    // scalar gates travel as raw bf16 bits in registers of threads 0..63, loaded
    // one chunk ahead from a clamped address and converted when the chunk starts
    unsigned short g_a = 0, g_b = 0, g_w = 0;
    auto load_scalar_gates = [&](int ci) {
        if (tid < C) {
            const int t = min(ci * C + tid, T - 1);
            const size_t gi = ((size_t)bb * T + t) * H + h;
            if (p.akind == GDR_GATE_SCALAR) g_a = ((const unsigned short*)p.alpha)[gi];
            if (p.bkind == GDR_GATE_SCALAR) g_b = ((const unsigned short*)p.bg)[gi];
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
        const uint32_t vbuf = sbase + OFF_V + (ci & 1) * 8192u;
        GDR_TRACE(0);
        // ---- scalar gates of this chunk (loaded one chunk ahead) -----------
        if (tid < C) {
            const bool valid = t0 + tid < T;
            s_ascal[tid] = (p.akind == GDR_GATE_SCALAR && valid) ? bits_to_f32(g_a) : 1.f;
            s_bscal[tid] = (p.bkind == GDR_GATE_SCALAR && valid) ? bits_to_f32(g_b) : 0.f;
            s_wscal[tid] = (p.wkind == GDR_GATE_SCALAR && valid) ? bits_to_f32(g_w)
                           : (p.wkind == GDR_GATE_NONE ? 1.f : 0.f);
        }
        GDR_WAIT(bar_tma, ph_tma);
        GDR_TRACE(1);

        // ---- build: log-decay scan and scaled operands --------------------
        // thread = (token group rg = warp: 8 tokens, channel group cg = lane: 4 channels);
        // a warp reads whole 256-byte token rows (conflict-free 8-byte pieces)
        {
            const int cg = tid & 31, rg = warp;
            const int ch0 = cg * 4;
            auto piece = [&](int r, int rows) {  // byte offset of channels ch0..ch0+3 of row r
                return sw128_chunk(r, cg >> 1, rows) + (uint32_t)(cg & 1) * 8u;
            };
            auto ld4 = [&](uint32_t base, int r, float* x4) {
                const uint2 u = *reinterpret_cast<const uint2*>(sm + base + piece(r, C));
                const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
                const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
                x4[0] = f0.x; x4[1] = f0.y; x4[2] = f1.x; x4[3] = f1.y;
            };
            auto st4 = [&](uint32_t base, int r, int rows, const float* x4) {
                uint2 u;
                u.x = pack_bf16x2(x4[0], x4[1]);
                u.y = pack_bf16x2(x4[2], x4[3]);
                *reinterpret_cast<uint2*>(sm + base + piece(r, rows)) = u;
            };
            float* scan = reinterpret_cast<float*>(sm + OFF_SCAN);  // [8 rg][128 ch] + [128]
            bool chunk_bad = false;  // decay span beyond the factorisation's range
            float lrow[8][4];  // channel decay: l_r - ref
            float aval[8][4];  // channel decay: alpha of this thread's tokens
            if (!ach) {
                // one decay per token: warp 0 scans the 64 tokens (2 per lane)
                if (warp == 0) {
                    const int lane = tid;
                    const float la0 = (2 * lane < n) ? lg2_approx(s_ascal[2 * lane]) : 0.f;
                    const float la1 = (2 * lane + 1 < n) ? lg2_approx(s_ascal[2 * lane + 1]) : 0.f;
                    float x = la0 + la1;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        float y = __shfl_up_sync(0xffffffffu, x, off);
                        if (lane >= off) x += y;
                    }
                    const float l1 = x, l0v = x - la1;  // inclusive prefix at tokens 2 lane + 1, 2 lane
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
                    ld4(OFF_GA, r, aval[i]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if (r >= n) aval[i][e] = 1.f;  // padding tokens do not decay
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
                    ref[e] = 0.5f * (l0[e] + tot[e]);  // tot = l_{n-1} (padding adds 0)
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
            }
            if (__syncthreads_or(chunk_bad)) {
                // the chunk's decay ratios do not fit two bounded factors: apply
                // its tokens one by one (fp32, raw inputs), then go on
                if (tid == 0) flag_status(p.d_status, GDR_DEVICE_DECAY_RANGE);
                if (tid == 0 && ci + 1 < nchunks) issue_loads(ci + 1);
                if (ci + 1 < nchunks) load_scalar_gates(ci + 1);
                const ExactArgs ex{(const __nv_bfloat16*)p.q, (const __nv_bfloat16*)p.k,
                                   (const __nv_bfloat16*)p.v, (const __nv_bfloat16*)p.alpha,
                                   (const __nv_bfloat16*)p.bg, (const __nv_bfloat16*)p.wg,
                                   p.akind, p.bkind, p.wkind, p.o, T, H, H / p.group, p.dv};
                exact_tokens(ex, S, reinterpret_cast<float*>(sm + OFF_U), bb, h, hq, v0, t0, n, tid);
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) st_chunk(sm + OFF_SBF, sw128_chunk(row, wg * 4 + ch, DK), &S[8 * ch]);
                fence_proxy_async();
                tc_fence_before();
                __syncthreads();
                continue;
            }
            float rowf_c[4];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = rg * 8 + i;
                float k4[4], q4[4], b4[4], w4[4];
                ld4(OFF_KIN, r, k4);
                ld4(OFF_QIN, r, q4);
                if (bch) ld4(OFF_GB, r, b4);
                else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) b4[e] = s_bscal[r];
                }
                if (!TIED) {
                    if (p.wkind == GDR_GATE_TIED) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) w4[e] = b4[e];
                    } else if (wch) {
                        ld4(OFF_GW, r, w4);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) w4[e] = s_wscal[r];
                    }
                }
                float rop_k[4], rop_q[4], cop_k[4], cop_w[4];
                const bool valid = r < n;
                const float rs = ach ? 0.f : s_rowf[r], cs = ach ? 0.f : s_colf[r];
                if (ach) {
                    // rowf by a multiply chain over this thread's 8 tokens (one exp2 per
                    // chain), colf = 1 / rowf by Newton iterations on the FMA pipe
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        rowf_c[e] = (i == 0) ? ex2_approx(lrow[0][e]) : rowf_c[e] * aval[i][e];
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float rowf = ach ? rowf_c[e] : rs;
                    const float colf = ach ? rcp_newton(rowf) : cs;
                    const float kk = valid ? k4[e] : 0.f;
                    const float qq = valid ? q4[e] : 0.f;
                    rop_k[e] = b4[e] * kk * rowf;
                    rop_q[e] = qq * rowf;
                    cop_k[e] = kk * colf;
                    cop_w[e] = TIED ? 0.f : w4[e] * kk * colf;
                }
                st4(OFF_ROP, r, 128, rop_k);
                st4(OFF_ROP, 64 + r, 128, rop_q);
                st4(OFF_COP, r, N1, cop_k);
                if (!TIED) st4(OFF_COP, 64 + r, N1, cop_w);
            }
        }
        GDR_BEFORE_MMA();
        GDR_TRACE(2);

        // ---- P1: D1 = [Kb ; Qs] x [Ks ; Kws]^T --------------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, N1, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t koff = (ks >> 2) * 16384u + (ks & 3) * 32u;
                const uint32_t koffb = (ks >> 2) * (uint32_t)(N1 * 128) + (ks & 3) * 32u;
                mma_bf16(tmem + TM_D1, sdesc_sw128(sbase + OFF_ROP + koff, 16, 1024),
                         sdesc_sw128(sbase + OFF_COP + koffb, 16, 1024), id, ks > 0);
            }
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        GDR_TRACE(3);

        // ---- unload D1 (each warpgroup one half of the columns): A (fp32),
        //      Aq -> AQ rows 64..127; general gates: Bm -> X, Bq -> APRE rows 64..127 ----
        {
            const int r = row & 63;
            float d[32], d2[32];
            tmem_ld32_async(tmem + lane_base + TM_D1 + wg * 32, d);
            if (!TIED) tmem_ld32_async(tmem + lane_base + TM_D1 + 64 + wg * 32, d2);
            tmem_wait_ld();
            if (row < 64) {
                float* A32 = reinterpret_cast<float*>(sm + OFF_A32);
#pragma unroll
                for (int j4 = 0; j4 < 32; j4 += 4) {
                    const int j = wg * 32 + j4;
                    float4 x = make_float4(j < r ? d[j4] : 0.f, j + 1 < r ? d[j4 + 1] : 0.f,
                                           j + 2 < r ? d[j4 + 2] : 0.f, j + 3 < r ? d[j4 + 3] : 0.f);
                    *reinterpret_cast<float4*>(f32_at(A32, r, j)) = x;
                }
                // transposed diagonal block: AT[I][j][rr] = A[16 I + rr][16 I + j]
                const int I = r >> 4, rr = r & 15;
                if ((I >> 1) == wg) {
                    float* at = reinterpret_cast<float*>(sm + OFF_P32) + I * 272;
                    // the block's 16 columns start at d[0] (even I) or d[16] (odd I)
                    if (I & 1) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) at[j * 16 + rr] = j < rr ? d[16 + j] : 0.f;
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) at[j * 16 + rr] = j < rr ? d[j] : 0.f;
                    }
                }
            } else {
                float x[8];
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = (wg * 32 + c8 * 8 + e <= r) ? d[c8 * 8 + e] : 0.f;
                    st_chunk(sm + OFF_AQ, sw128_chunk(row, wg * 4 + c8, 128), x);
                }
            }
            if (!TIED) {
                float x[8];
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = wg * 32 + c8 * 8 + e;
                        x[e] = (row < 64 ? j < r : j <= r) ? d2[c8 * 8 + e] : 0.f;
                    }
                    if (row < 64) st_chunk(sm + OFF_X, sw128_chunk(r, wg * 4 + c8, 64), x);   // Bm
                    else st_chunk(sm + OFF_APRE, sw128_chunk(row, wg * 4 + c8, 128), x);     // Bq
                }
            }
        }
        __syncthreads();
        GDR_TRACE(4);

        // ---- solve T = (I + A)^-1 (fp32) by recursive halving:
        //      16x16 diagonal blocks by forward substitution, then
        //      T_(I+1)I = -T_(I+1)(I+1) A_(I+1)I T_II for the pairs (1,0), (3,2),
        //      then T_bot,top = -T_bot A_bot,top T_top for the 32x32 halves ----------
        {
            float* A32 = reinterpret_cast<float*>(sm + OFF_A32);
            float* T32 = reinterpret_cast<float*>(sm + OFF_T32);
            solve_unit_lower(A32, T32, reinterpret_cast<float*>(sm + OFF_P32), tid, warp);
            GDR_TRACE(14);
            // L = [T ; 0] (bf16, 128 x 64); tied: APRE rows 0..63 = T Diag(beta).
            // Thread (row r = tid & 63, half = tid >> 6 of 4): chunks 2*half, 2*half+1.
            {
                const int r = tid & 63, q4 = tid >> 6;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int c8 = q4 * 2 + cc;
                    float x[8];
#pragma unroll
                    for (int e4 = 0; e4 < 8; e4 += 4) {
                        const int j = c8 * 8 + e4;
                        // T is lower triangular: the upper-right 32x32 block is zero
                        float4 t4 = (j < 32 || r >= 32)
                                        ? *reinterpret_cast<const float4*>(f32_at(T32, r, j))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                        x[e4] = t4.x; x[e4 + 1] = t4.y; x[e4 + 2] = t4.z; x[e4 + 3] = t4.w;
                    }
                    st_chunk(sm + OFF_L, sw128_chunk(r, c8, 128), x);
                    st_zero_chunk(sm + OFF_L, sw128_chunk(64 + r, c8, 128));
                    if (TIED) {
                        const float4 b0 = *reinterpret_cast<const float4*>(s_bscal + c8 * 8);
                        const float4 b1 = *reinterpret_cast<const float4*>(s_bscal + c8 * 8 + 4);
                        x[0] *= b0.x; x[1] *= b0.y; x[2] *= b0.z; x[3] *= b0.w;
                        x[4] *= b1.x; x[5] *= b1.y; x[6] *= b1.z; x[7] *= b1.w;
                        st_chunk(sm + OFF_APRE, sw128_chunk(r, c8, 128), x);
                    }
                }
            }
        }
        GDR_BEFORE_MMA();
        GDR_TRACE(5);

        // ---- P2: D2 = [T ; 0] x [Kb | Bm];  tied: P3 D3 = [T Diag(beta) ; 0] x V ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idW = idesc_bf16(128, 128, 0, 1);
            const uint32_t id64 = idesc_bf16(128, 64, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = sdesc_sw128(sbase + OFF_L + ks * 32u, 16, 1024);
                mma_bf16(tmem + TM_D2, ad, sdesc_sw128(sbase + OFF_ROP + ks * 2048u, 16384, 1024), idW, ks > 0);
                if (!TIED)
                    mma_bf16(tmem + TM_D2 + 128, ad, sdesc_sw128(sbase + OFF_X + ks * 2048u, 8192, 1024), id64, ks > 0);
            }
            if (TIED) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_D3, sdesc_sw128(sbase + OFF_APRE + ks * 32u, 16, 1024),
                             sdesc_sw128(vbuf + ks * 2048u, 8192, 1024), id64, ks > 0);
            }
            mma_commit(bar_mma);
        }
        // ---- while P2 runs: Qs.2^ref in place (rows 64..127 of [Kb ; Qs], not read by P2)
        auto load_eref = [&](int c0, float* er) {
            if (ach) {
                const float4 e0 = *reinterpret_cast<const float4*>(s_eref + c0);
                const float4 e1 = *reinterpret_cast<const float4*>(s_eref + c0 + 4);
                er[0] = e0.x; er[1] = e0.y; er[2] = e0.z; er[3] = e0.w;
                er[4] = e1.x; er[5] = e1.y; er[6] = e1.z; er[7] = e1.w;
            } else {
                const float e = s_eref[0];
#pragma unroll
                for (int i = 0; i < 8; ++i) er[i] = e;
            }
        };
        if (row >= 64) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int ch = wg * 8 + c;
                float x[8], er[8];
                const uint32_t off = sw128_chunk(row, ch, 128);
                ld_chunk(sm + OFF_ROP, off, x);
                load_eref(ch * 8, er);
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] *= er[e];
                st_chunk(sm + OFF_ROP, off, x);
            }
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        GDR_TRACE(6);
        // the input region (A, T, L, Bm) is free: prefetch the next chunk
        if (tid == 0 && ci + 1 < nchunks) issue_loads(ci + 1);
        if (ci + 1 < nchunks) load_scalar_gates(ci + 1);

        // ---- W -> -W.2^ref in place of Kb (rows 0..63); general: -T Bm -> APRE -----
        if (row < 64) {
            float d[32], d1[32], d2[32];
            tmem_ld32_async(tmem + lane_base + TM_D2 + wg * 64, d);
            tmem_ld32_async(tmem + lane_base + TM_D2 + wg * 64 + 32, d1);
            if (!TIED) tmem_ld32_async(tmem + lane_base + TM_D2 + 128 + wg * 32, d2);
            tmem_wait_ld();
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                const int col = wg * 64 + cb * 32;
                const float* dd = cb ? d1 : d;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    float x[8], er[8];
                    load_eref(col + c4 * 8, er);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = -dd[c4 * 8 + e] * er[e];
                    st_chunk(sm + OFF_ROP, sw128_chunk(row, col / 8 + c4, 128), x);
                }
            }
            if (!TIED) {
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = -d2[c4 * 8 + e];
                    st_chunk(sm + OFF_APRE, sw128_chunk(row, wg * 4 + c4, 128), x);
                }
            }
        }
        GDR_BEFORE_MMA();
        GDR_TRACE(7);

        // ---- general: P3 D3 = [-T Bm ; Bq] x V;  S1: D3 += [-W ; Qs.2^ref] x S -----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id64 = idesc_bf16(128, NV, 0, 1);
            if (!TIED) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_D3, sdesc_sw128(sbase + OFF_APRE + ks * 32u, 16, 1024),
                             sdesc_sw128(vbuf + ks * 2048u, 8192, 1024), id64, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(tmem + TM_D3, sdesc_sw128(sbase + OFF_ROP + (ks >> 2) * 16384u + (ks & 3) * 32u, 16, 1024),
                         sdesc_sw128(sbase + OFF_SBF + ks * 2048u, 8192, 1024), id64, 1);
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        GDR_TRACE(8);

        // ---- U (rows 0..63 of D3) -> bf16 ---------------------------------------
        if (row < 64) {
            float d[32];
            tmem_ld32(tmem + lane_base + TM_D3 + wg * 32, d);
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) st_chunk(sm + OFF_U, sw128_chunk(row, wg * 4 + c8, 64), d + 8 * c8);
        }
        GDR_BEFORE_MMA();
        GDR_TRACE(9);

        // ---- S2: D3 += [0 ; Aq] x U ;  D4 = [Ks ; Kws]^T x [U ; V] -----------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idK = idesc_bf16(128, NV, 0, 1);
            const uint32_t idM = idesc_bf16(128, NV, 1, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + TM_D3, sdesc_sw128(sbase + OFF_AQ + ks * 32u, 16, 1024),
                         sdesc_sw128(sbase + OFF_U + ks * 2048u, 8192, 1024), idK, 1);
#pragma unroll
            for (int ks = 0; ks < N1 / 16; ++ks) {
                const uint64_t ad = sdesc_sw128(sbase + OFF_COP + ks * 2048u, N1 * 128, 1024);
                const uint64_t bd = ks < 4 ? sdesc_sw128(sbase + OFF_U + ks * 2048u, 8192, 1024)
                                           : sdesc_sw128(vbuf + (ks - 4) * 2048u, 8192, 1024);
                mma_bf16(tmem + TM_D4, ad, bd, idM, ks > 0);
            }
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        GDR_TRACE(10);

        // ---- O (rows 64..127 of D3) -> global; state update from D4 -----------------
        {
            float d[32], dS[32];
            if (row >= 64) tmem_ld32_async(tmem + lane_base + TM_D3 + wg * 32, d);
            tmem_ld32_async(tmem + lane_base + TM_D4 + wg * 32, dS);
            tmem_wait_ld();
            if (row >= 64) {
                const int t = t0 + row - 64;
                if (t < T) {
                    __nv_bfloat16* op = p.o + (((size_t)bb * T + t) * H + h) * p.dv + v0 + wg * 32;
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
            const float gC = s_gC[row], fS = s_fS[row];
#pragma unroll
            for (int j = 0; j < NH; ++j) S[j] = gC * S[j] + fS * dS[j];
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) st_chunk(sm + OFF_SBF, sw128_chunk(row, wg * 4 + ch, DK), &S[8 * ch]);
        }
        tc_fence_before();
        __syncthreads();
        GDR_TRACE(11);
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

// ---------------------------------------------------------------------------
// Gated DeltaNet form: scalar decay per token, tied scalar b = w = beta.
// Every scale factor is per token, so it folds into MMA outputs or into the
// small T-derived operands and the raw q / k tiles from TMA are the MMA
// operands (no operand build):
//   A  = Diag(beta) ((K K^T) . G)            (strict lower)     [D1 unload]
//   Aq = (Q K^T) . G                         (lower)            [D1 unload]
//   W  = T Diag(beta g) K                     (P2, A = [T Diag(beta g) ; 0])
//   U  = T Diag(beta) V - W S                 (P3 pre-load + S1)
//   O  = Diag(g) (Q S) + Aq U                 (S1 gives Q S, S2 gives Aq U)
//   S' = g_{n-1} S + (Diag(g_{n-1}/g) K)^T U  (K copy scaled per token, S2)
// with g_r = 2^l_r and G_rj = g_r / g_j = 2^(l_r - l_j), formed per element on
// the unload (at most 1 wherever it is used, so every alpha in (0, 1] is in range).
// Inputs are double-buffered: the next chunk's TMA is issued as a chunk starts.
namespace gdn {
constexpr uint32_t OFF_QK = 0;          // [K ; Q] bf16 [128 x 128], 2 buffers; rows 0..63 become -W
constexpr uint32_t OFF_K2 = 65536;      // K bf16 [64 x 128], 2 buffers; scaled by g_{n-1}/g per token
constexpr uint32_t OFF_V = 98304;       // V slice bf16 [64 x 64], 2 buffers
constexpr uint32_t OFF_L = 114688;      // [T Diag(beta g) ; 0] bf16 [128 x 64]
constexpr uint32_t OFF_APRE = 131072;   // [T Diag(beta) ; 0] bf16 [128 x 64]
constexpr uint32_t OFF_AQ = 147456;     // [0 ; Aq] bf16 [128 x 64]
constexpr uint32_t OFF_SBF = 163840;    // S bf16 [128 x 64]
constexpr uint32_t OFF_U = 180224;      // U bf16 [64 x 64]
constexpr uint32_t OFF_A32 = 188416;    // A fp32 [64 x 64]
constexpr uint32_t OFF_T32 = 204800;    // T fp32 [64 x 64]
constexpr uint32_t OFF_SCR = 221184;    // solve scratch fp32 (5 KB)
constexpr uint32_t OFF_SMALL = 226304;  // per-token scalars, barriers
constexpr uint32_t SMEM_BYTES = OFF_SMALL + 3072 + 1024;
constexpr uint32_t TM_D1 = 0, TM_D2 = 64, TM_D3 = 192, TM_D4 = 256, TM_D5 = 320, TM_COLS = 512;
}  // namespace gdn

__global__ void __launch_bounds__(NT, 1) chunk_fwd_gdn_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int wg = warp >> 2;
    const int row = tid & 127;
    const int vt = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int hq = h / p.group;  // q / k head of this value head
    const int v0 = vt * NV;
    const int T = p.T, H = p.H;
    const int nchunks = (T + C - 1) / C;

    // per-token factors, double-buffered by chunk parity (the next chunk's are
    // computed while the current chunk's last MMA runs): [2][64] each
    float* s_beta2 = reinterpret_cast<float*>(sm + gdn::OFF_SMALL);
    float* s_l2 = s_beta2 + 128;   // [2][64] log2 prefix of alpha over the chunk
    float* s_g2 = s_beta2 + 384;
    float* s_gcr2 = s_beta2 + 512;
    float* s_misc2 = s_beta2 + 640;   // [2][4]: g_{n-1}
    float* s_alpha = s_beta2 + 648;   // [64] staging of the next chunk's decays
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + gdn::OFF_SMALL + 2880);  // [2]
    uint64_t* bar_mma = bar_tma + 2;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + gdn::OFF_SMALL + 2912);
    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) tmem_alloc(s_tmem, gdn::TM_COLS);
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
        uint8_t* qk = sm + gdn::OFF_QK + buf * 32768;
        uint8_t* k2 = sm + gdn::OFF_K2 + buf * 16384;
        mbar_expect_tx(&bar_tma[buf], 7u * 8192u);
        // [K ; Q]: each 64-column block holds 128 rows (k rows 0..63, q rows 64..127)
        tma_load_4d(qk, &tm_k, &bar_tma[buf], 0, hq, t0, bb);
        tma_load_4d(qk + 16384, &tm_k, &bar_tma[buf], 64, hq, t0, bb);
        tma_load_4d(qk + 8192, &tm_q, &bar_tma[buf], 0, hq, t0, bb);
        tma_load_4d(qk + 16384 + 8192, &tm_q, &bar_tma[buf], 64, hq, t0, bb);
        tma_load_4d(k2, &tm_k, &bar_tma[buf], 0, hq, t0, bb);
        tma_load_4d(k2 + 8192, &tm_k, &bar_tma[buf], 64, hq, t0, bb);
        tma_load_4d(sm + gdn::OFF_V + buf * 8192, &tm_v, &bar_tma[buf], v0, h, t0, bb);
    };

    // ---- initial state; constant zero blocks ----------------------------------
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
        for (int ch = 0; ch < 4; ++ch) st_chunk(sm + gdn::OFF_SBF, sw128_chunk(row, wg * 4 + ch, DK), &S[8 * ch]);
        if (tid < 64) {  // AQ rows 0..63, L and APRE rows 64..127 stay zero
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                st_zero_chunk(sm + gdn::OFF_AQ, sw128_chunk(tid, ch, 128));
                st_zero_chunk(sm + gdn::OFF_L, sw128_chunk(64 + tid, ch, 128));
                st_zero_chunk(sm + gdn::OFF_APRE, sw128_chunk(64 + tid, ch, 128));
            }
        }
    }
    unsigned short g_a = 0, g_b = 0;
    auto load_scalar_gates = [&](int ci) {
        if (tid < C) {
            const int t = min(ci * C + tid, T - 1);
            const size_t gi = ((size_t)bb * T + t) * H + h;
            g_a = ((const unsigned short*)p.alpha)[gi];
            g_b = ((const unsigned short*)p.bg)[gi];
        }
    };
    auto bits_to_f32 = [](unsigned short u) { return __uint_as_float((uint32_t)u << 16); };
    // one warp: prefix sum of log2 alpha over the chunk's 64 tokens (2 per lane),
    // then the bounded factors around the reference and the decay products
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
        const float last = __shfl_sync(0xffffffffu, l1, 31);
        float* l = s_l2 + par * 64;
        float* g = s_g2 + par * 64;
        float* gcr = s_gcr2 + par * 64;
        l[2 * lane] = l0v;
        l[2 * lane + 1] = l1;
        g[2 * lane] = ex2_approx(l0v);
        g[2 * lane + 1] = ex2_approx(l1);
        gcr[2 * lane] = ex2_approx(last - l0v);
        gcr[2 * lane + 1] = ex2_approx(last - l1);
        if (lane == 0) s_misc2[par * 4] = ex2_approx(last);
    };
    // stage chunk ci's gates (threads 0..63 hold them in g_a, g_b)
    auto stage_gates = [&](int ci) {
        if (tid < C) {
            const bool valid = ci * C + tid < T;
            s_alpha[tid] = valid ? bits_to_f32(g_a) : 1.f;
            s_beta2[(ci & 1) * 64 + tid] = valid ? bits_to_f32(g_b) : 0.f;
        }
    };
    if (tid == 0 && nchunks > 0) issue_loads(0);
    if (nchunks > 0) {
        load_scalar_gates(0);
        stage_gates(0);
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
        const int n = min(C, T - t0);
        const int buf = ci & 1;
        const uint32_t qkb = sbase + gdn::OFF_QK + buf * 32768u;
        const uint32_t k2b = sbase + gdn::OFF_K2 + buf * 16384u;
        const uint32_t vbuf = sbase + gdn::OFF_V + buf * 8192u;
        GDR_TRACE(0);
        if (tid == 0 && ci + 1 < nchunks) issue_loads(ci + 1);  // its buffers were freed by chunk ci-1
        if (ci + 1 < nchunks) load_scalar_gates(ci + 1);         // consumed before S2 of this chunk
        const int par = ci & 1;
        const float* s_beta = s_beta2 + par * 64;
        const float* s_l = s_l2 + par * 64;
        const float* s_g = s_g2 + par * 64;
        const float* s_gcr = s_gcr2 + par * 64;
        const float* s_misc = s_misc2 + par * 4;
        if (buf == 0) GDR_WAIT(&bar_tma[0], ph_tma0);
        else GDR_WAIT(&bar_tma[1], ph_tma1);
        GDR_TRACE(1);
        GDR_TRACE(2);

        // ---- P1: D1 = [K ; Q] x K^T -----------------------------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t koff = (ks >> 2) * 16384u + (ks & 3) * 32u;
                mma_bf16(tmem + gdn::TM_D1, sdesc_sw128(qkb + koff, 16, 1024), sdesc_sw128(qkb + koff, 16, 1024),
                         id, ks > 0);
            }
            mma_commit(bar_mma);
        }
        // while P1 runs: scale the K copy's rows by g_{n-1} / g_r (rows of S2's operand)
        {
            const int r = tid >> 2, c4 = (tid & 3) * 4;  // 64 rows x 4 threads x 4 chunks
            const float f = s_gcr[r];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float x[8];
                const uint32_t off = sw128_chunk(r, c4 + cc, 64);
                ld_chunk(sm + gdn::OFF_K2 + buf * 16384, off, x);
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] *= f;
                st_chunk(sm + gdn::OFF_K2 + buf * 16384, off, x);
            }
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        GDR_TRACE(3);

        // ---- unload D1: A (fp32) and its transposed diagonal blocks; Aq -> AQ ---------
        {
            const int r = row & 63;
            float d[32];
            tmem_ld32(tmem + lane_base + gdn::TM_D1 + wg * 32, d);
            // decay ratio g_r / g_j = 2^(l_r - l_j) per element (at most 1 where used)
            const float rf = row < 64 ? s_beta[r] : 1.f, lr = s_l[r];
            float cf[32];
#pragma unroll
            for (int j4 = 0; j4 < 32; j4 += 4) {
                const float4 l4 = *reinterpret_cast<const float4*>(s_l + wg * 32 + j4);
                cf[j4] = ex2_approx(fminf(lr - l4.x, 0.f));
                cf[j4 + 1] = ex2_approx(fminf(lr - l4.y, 0.f));
                cf[j4 + 2] = ex2_approx(fminf(lr - l4.z, 0.f));
                cf[j4 + 3] = ex2_approx(fminf(lr - l4.w, 0.f));
            }
            if (row < 64) {
                float* A32 = reinterpret_cast<float*>(sm + gdn::OFF_A32);
#pragma unroll
                for (int j4 = 0; j4 < 32; j4 += 4) {
                    const int j = wg * 32 + j4;
                    float4 x;
                    x.x = j < r ? rf * cf[j4] * d[j4] : 0.f;
                    x.y = j + 1 < r ? rf * cf[j4 + 1] * d[j4 + 1] : 0.f;
                    x.z = j + 2 < r ? rf * cf[j4 + 2] * d[j4 + 2] : 0.f;
                    x.w = j + 3 < r ? rf * cf[j4 + 3] * d[j4 + 3] : 0.f;
                    d[j4] = x.x; d[j4 + 1] = x.y; d[j4 + 2] = x.z; d[j4 + 3] = x.w;
                    *reinterpret_cast<float4*>(f32_at(A32, r, j)) = x;
                }
                const int I = r >> 4, rr = r & 15;
                if ((I >> 1) == wg) {
                    float* at = reinterpret_cast<float*>(sm + gdn::OFF_SCR) + I * 272;
                    if (I & 1) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) at[j * 16 + rr] = d[16 + j];
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) at[j * 16 + rr] = d[j];
                    }
                }
            } else {
                float x[8];
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int jl = c8 * 8 + e;
                        x[e] = (wg * 32 + jl <= r) ? rf * cf[jl] * d[jl] : 0.f;
                    }
                    st_chunk(sm + gdn::OFF_AQ, sw128_chunk(row, wg * 4 + c8, 128), x);
                }
            }
        }
        __syncthreads();
        GDR_TRACE(4);

        // ---- solve; L = T Diag(beta g), APRE = T Diag(beta) (rows 0..63) ------------
        {
            float* A32 = reinterpret_cast<float*>(sm + gdn::OFF_A32);
            float* T32 = reinterpret_cast<float*>(sm + gdn::OFF_T32);
            solve_unit_lower(A32, T32, reinterpret_cast<float*>(sm + gdn::OFF_SCR), tid, warp);
            GDR_TRACE(14);
            const int r = tid & 63, q4 = tid >> 6;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c8 = q4 * 2 + cc;
                float x[8], y[8];
#pragma unroll
                for (int e4 = 0; e4 < 8; e4 += 4) {
                    const int j = c8 * 8 + e4;
                    float4 t4 = (j < 32 || r >= 32) ? *reinterpret_cast<const float4*>(f32_at(T32, r, j))
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float4 b4 = *reinterpret_cast<const float4*>(s_beta + j);
                    const float4 g4 = *reinterpret_cast<const float4*>(s_g + j);
                    y[e4] = t4.x * b4.x; y[e4 + 1] = t4.y * b4.y; y[e4 + 2] = t4.z * b4.z; y[e4 + 3] = t4.w * b4.w;
                    x[e4] = y[e4] * g4.x; x[e4 + 1] = y[e4 + 1] * g4.y; x[e4 + 2] = y[e4 + 2] * g4.z;
                    x[e4 + 3] = y[e4 + 3] * g4.w;
                }
                st_chunk(sm + gdn::OFF_L, sw128_chunk(r, c8, 128), x);
                st_chunk(sm + gdn::OFF_APRE, sw128_chunk(r, c8, 128), y);
            }
        }
        GDR_BEFORE_MMA();
        GDR_TRACE(5);

        // ---- P2: D2 = [T Diag(beta g) ; 0] x K;  P3: D3 = [T Diag(beta) ; 0] x V ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idW = idesc_bf16(128, 128, 0, 1);
            const uint32_t id64 = idesc_bf16(128, 64, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + gdn::TM_D2, sdesc_sw128(sbase + gdn::OFF_L + ks * 32u, 16, 1024),
                         sdesc_sw128(qkb + ks * 2048u, 16384, 1024), idW, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + gdn::TM_D3, sdesc_sw128(sbase + gdn::OFF_APRE + ks * 32u, 16, 1024),
                         sdesc_sw128(vbuf + ks * 2048u, 8192, 1024), id64, ks > 0);
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        GDR_TRACE(6);

        // ---- -W -> rows 0..63 of [K ; Q] (K is no longer read from this tile) ----------
        if (row < 64) {
            float d[32], d1[32];
            tmem_ld32_async(tmem + lane_base + gdn::TM_D2 + wg * 64, d);
            tmem_ld32_async(tmem + lane_base + gdn::TM_D2 + wg * 64 + 32, d1);
            tmem_wait_ld();
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                const int col = wg * 64 + cb * 32;
                const float* dd = cb ? d1 : d;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = -dd[c4 * 8 + e];
                    st_chunk(sm + gdn::OFF_QK + buf * 32768, sw128_chunk(row, col / 8 + c4, 128), x);
                }
            }
        }
        GDR_BEFORE_MMA();
        GDR_TRACE(7);

        // ---- S1: D3 += [-W ; Q] x S ------------------------------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id64 = idesc_bf16(128, NV, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(tmem + gdn::TM_D3, sdesc_sw128(qkb + (ks >> 2) * 16384u + (ks & 3) * 32u, 16, 1024),
                         sdesc_sw128(sbase + gdn::OFF_SBF + ks * 2048u, 8192, 1024), id64, 1);
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        GDR_TRACE(8);

        // ---- U (rows 0..63 of D3) -> bf16 -------------------------------------------
        if (row < 64) {
            float d[32];
            tmem_ld32(tmem + lane_base + gdn::TM_D3 + wg * 32, d);
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) st_chunk(sm + gdn::OFF_U, sw128_chunk(row, wg * 4 + c8, 64), d + 8 * c8);
        }
        if (ci + 1 < nchunks) stage_gates(ci + 1);
        GDR_BEFORE_MMA();
        GDR_TRACE(9);

        // ---- S2: D5 = [0 ; Aq] x U ;  D4 = (Diag(g_{n-1}/g) K)^T x U ------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idK = idesc_bf16(128, NV, 0, 1);
            const uint32_t idM = idesc_bf16(128, NV, 1, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                mma_bf16(tmem + gdn::TM_D5, sdesc_sw128(sbase + gdn::OFF_AQ + ks * 32u, 16, 1024),
                         sdesc_sw128(sbase + gdn::OFF_U + ks * 2048u, 8192, 1024), idK, ks > 0);
                mma_bf16(tmem + gdn::TM_D4, sdesc_sw128(k2b + ks * 2048u, 8192, 1024),
                         sdesc_sw128(sbase + gdn::OFF_U + ks * 2048u, 8192, 1024), idM, ks > 0);
            }
            mma_commit(bar_mma);
        }
        if (warp == 7 && ci + 1 < nchunks) decay_scan(ci + 1, tid & 31);  // overlaps S2
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        GDR_TRACE(10);

        // ---- O = g Q S + Aq U (rows 64..127) -> global; S = g_{n-1} S + D4 ----------
        {
            float d[32], d5[32], dS[32];
            if (row >= 64) {
                tmem_ld32_async(tmem + lane_base + gdn::TM_D3 + wg * 32, d);
                tmem_ld32_async(tmem + lane_base + gdn::TM_D5 + wg * 32, d5);
            }
            tmem_ld32_async(tmem + lane_base + gdn::TM_D4 + wg * 32, dS);
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
            for (int ch = 0; ch < 4; ++ch) st_chunk(sm + gdn::OFF_SBF, sw128_chunk(row, wg * 4 + ch, DK), &S[8 * ch]);
        }
        tc_fence_before();
        __syncthreads();
        GDR_TRACE(11);
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
    if (warp == 0) tmem_dealloc(tmem, gdn::TM_COLS);
#undef GDR_WAIT
#undef GDR_BEFORE_MMA
}

}  // namespace chunk

// Host-side launch (tensor maps are built by the caller).
cudaError_t launch_chunk_sm100(const CUtensorMap* maps, const void* q, const void* k, const void* v,
                               const void* alpha, const void* b,
                               const void* w, int akind, int bkind, int wkind, bool tied,
                               const float* S0, void* o, float* ST, int* d_status, int B, int T,
                               int H, int dv, int group, cudaStream_t st) {
    chunk::Params p;
    p.q = q; p.k = k; p.v = v;
    p.alpha = alpha; p.bg = b; p.wg = w;
    p.S0 = S0; p.o = (__nv_bfloat16*)o; p.ST = ST; p.d_status = d_status;
    p.B = B; p.T = T; p.H = H; p.dv = dv;
    p.akind = akind; p.bkind = bkind; p.wkind = wkind;
    p.group = group;
    dim3 grid(dv / chunk::NV, H, B);
    const bool ach = akind == GDR_GATE_CHANNEL;
    auto launch = [&](auto kern) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, chunk::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        kern<<<grid, chunk::NT, chunk::SMEM_BYTES, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], p);
        return cudaSuccess;
    };
    cudaError_t e;
    if (tied && akind == GDR_GATE_SCALAR) {
        e = cudaFuncSetAttribute(chunk::chunk_fwd_gdn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, chunk::gdn::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        chunk::chunk_fwd_gdn_kernel<<<grid, chunk::NT, chunk::gdn::SMEM_BYTES, st>>>(maps[0], maps[1], maps[2], p);
    } else if (tied) e = ach ? launch(chunk::chunk_fwd_kernel<true, true>) : launch(chunk::chunk_fwd_kernel<true, false>);
    else e = ach ? launch(chunk::chunk_fwd_kernel<false, true>) : launch(chunk::chunk_fwd_kernel<false, false>);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace gdr

#ifdef GDR_TRACE_PHASES
extern "C" int gdr_trace_read(unsigned long long* host, int n) {
    return (int)cudaMemcpyFromSymbol(host, gdr::chunk::g_trace, sizeof(unsigned long long) * n);
}
#endif
