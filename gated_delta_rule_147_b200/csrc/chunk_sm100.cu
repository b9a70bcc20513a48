// Chunkwise-parallel gated delta-rule forward on sm_100a tensor cores.
//
// Math (per head, chunk of C = 64 tokens r = 0..n-1, state S at chunk start;
// "Recurrent Memory: Write, Erase, Decay, Read" sections 03-05 for the
// reassociation into chunks and the prefix sum of log decays; "Erase-then-
// Delta Attention" abstract for the chunkwise WY form with the decay absorbed
// into the erase factors):
//   l_r   = sum_{j<=r} log2 alpha_j (per channel), g_r = 2^l_r
//   ref   = (l_0 + l_{n-1}) / 2 per channel; rowf_r = 2^(l_r - ref),
//           colf_r = 2^(ref - l_r) (so rowf_r colf_j = g_r / g_j, both bounded)
//   A  = strict_lower[(b.k.rowf)(k.colf)^T]     Bm = strict_lower[(b.k.rowf)(w.k.colf)^T]
//   Aq = lower[(q.rowf)(k.colf)^T]              Bq = lower[(q.rowf)(w.k.colf)^T]
//   T  = (I + A)^-1                               (unit lower triangular solve)
//   E_top = T [b.k.g | Bm],  E_bot = [q.g | Bq] - Aq E_top
//   [-U ; O] = [E_top ; E_bot] [S ; V]            (O is the chunk's output)
//   S_new = Diag(g_{n-1}) S + Diag(2^(l_{n-1}-ref)) [(k.colf)^T U + (w.k.colf)^T V]
// With tied scalar gates b = w = beta, Bm = A Diag(beta) and the V columns
// simplify to E = [ [T b.k.g, -T Diag(beta)] ; [q.g - Aq T b.k.g, Aq T Diag(beta)] ],
// U becomes U + Diag(beta) V and the state update needs only (k.colf)^T U.
//
// One CTA (128 threads) owns one (batch, head, 64-column slice of d_v) and
// walks the chunks in order; the state slice stays on chip (fp32 registers,
// a bf16 copy in shared memory as the MMA operand). Per chunk five tcgen05
// MMAs run with fp32 accumulators in tensor memory:
//   P1  D1 = [b.k.rowf ; q.rowf] x [k.colf ; w.k.colf]^T        (A, Aq, Bm, Bq)
//   P2  D2 = [[T,0],[0,I]] x [ [b.k.g ; q.g] | X ]               (E_top, copy of bottom)
//   P3  D2 += [0 ; -Aq] x E_top                                  (E_bot)
//   S1  D3 = E x [S ; V]                                         (-U, O)
//   S2  D4 = [k.colf ; w.k.colf]^T x [U ; V]                     (state increment)
// q, k, v and channel gates arrive by TMA (128-byte swizzle) straight into
// the operand layout the MMAs read.
#include "common.cuh"

namespace gdr {
namespace chunk {

constexpr int C = 64;     // chunk length
constexpr int DK = 128;   // key dimension handled by this kernel
constexpr int NV = 64;    // value columns per CTA
constexpr int NT = 128;   // threads per CTA

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t OFF_QIN = 0;        // q chunk   [64 x 128] bf16, 2 column blocks of 8 KB
constexpr uint32_t OFF_KIN = 16384;    // k chunk
constexpr uint32_t OFF_GA = 32768;     // channel alpha chunk
constexpr uint32_t OFF_GB = 49152;     // channel b chunk
constexpr uint32_t OFF_GW = 65536;     // channel w chunk
//   after the operands are built the input region is reused:
constexpr uint32_t OFF_A32 = 0;        // A fp32 [64 x 64] (float4-swizzled rows)
constexpr uint32_t OFF_T32 = 16384;    // T fp32 [64 x 64]
constexpr uint32_t OFF_AP = 32768;     // [0 ; -Aq] bf16 [128 x 64]
constexpr uint32_t OFF_L = 49152;      // [[T,0],[0,I]] bf16 [128 x 128]
constexpr uint32_t OFF_V = 81920;      // v slice [64 x 64] bf16, two buffers of 8 KB
constexpr uint32_t OFF_ROP = 98304;    // [b.k.rowf ; q.rowf] bf16 [128 x 128]
constexpr uint32_t OFF_X = 131072;     // [Bm ; Bq] or [-Diag(beta) ; 0] bf16 [128 x 64]
constexpr uint32_t OFF_E = 98304;      // E bf16 [128 x 192] (over ROP and X, after P2)
constexpr uint32_t OFF_P32 = 98304;    // solve scratch fp32 3 x [16 x 16] (over ROP, after P1)
constexpr uint32_t OFF_SCAN = 131072;  // scan scratch fp32 (over X, during the build)
constexpr uint32_t OFF_RG = 147456;    // [b.k.g ; q.g] bf16 [128 x 128]
constexpr uint32_t OFF_U = 147456;     // U bf16 [64 x 64] (over RG, after P2)
constexpr uint32_t OFF_COP = 180224;   // [k.colf ; w.k.colf] bf16 [64 or 128 x 128]
constexpr uint32_t OFF_SBF = 212992;   // S bf16 [128 x 64]
constexpr uint32_t OFF_SMALL = 229376; // per-token scalars, per-channel factors, barriers
constexpr uint32_t SMEM_BYTES = 229376 + 2048 + 1024;  // + small area + alignment slack

// TMEM columns
constexpr uint32_t TM_D1 = 0, TM_D2 = 0, TM_D3 = 192, TM_D4 = 256, TM_COLS = 512;

struct Params {
    const void* alpha;  // scalar gates are read with plain loads
    const void* bg;
    const void* wg;
    const float* S0;
    __nv_bfloat16* o;
    float* ST;
    int* d_status;
    int B, T, H, dv;
    int akind, bkind, wkind;
};

__device__ __forceinline__ float ld_bf16_smem(const uint8_t* base, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + off));
}

// fp32 [64 x 64] scratch with rows of 16 float4 groups XOR-swizzled by row.
__device__ __forceinline__ float* f32_at(float* base, int r, int c) {
    return base + r * 64 + ((((c >> 2) ^ (r & 15))) << 2) + (c & 3);
}

__device__ __forceinline__ void st_chunk(uint8_t* base, uint32_t off, const float* x8) {
    uint4 u;
    u.x = pack_bf16x2(x8[0], x8[1]);
    u.y = pack_bf16x2(x8[2], x8[3]);
    u.z = pack_bf16x2(x8[4], x8[5]);
    u.w = pack_bf16x2(x8[6], x8[7]);
    *reinterpret_cast<uint4*>(base + off) = u;
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

template <bool TIED>
__global__ void __launch_bounds__(NT, 1) chunk_fwd_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
    const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_w,
    const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int vt = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int v0 = vt * NV;
    const int T = p.T, H = p.H;
    const int nchunks = (T + C - 1) / C;
    const bool ach = p.akind == GDR_GATE_CHANNEL, bch = p.bkind == GDR_GATE_CHANNEL,
               wch = p.wkind == GDR_GATE_CHANNEL;
    constexpr int N1 = TIED ? 64 : 128;  // rows of [k.colf ; w.k.colf]

    float* s_ascal = reinterpret_cast<float*>(sm + OFF_SMALL);          // [64] scalar alpha
    float* s_bscal = s_ascal + 64;                                       // [64] scalar b
    float* s_wscal = s_ascal + 128;                                      // [64] scalar w
    float* s_gC = s_ascal + 192;                                         // [128] g_{n-1}
    float* s_fS = s_ascal + 320;                                         // [128] 2^(l_{n-1}-ref)
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + OFF_SMALL + 1920);
    uint64_t* bar_mma = bar_tma + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + OFF_SMALL + 1936);
    int* s_flag = reinterpret_cast<int*>(sm + OFF_SMALL + 1940);

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
        *s_flag = 0;
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) tmem_alloc(s_tmem, TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    uint32_t ph_tma = 0, ph_mma = 0;
    bool ok = true;

    const uint32_t sbase = smem_u32(sm);
    auto issue_loads = [&](int ci) {
        const int t0 = ci * C;
        const uint32_t bytes = (uint32_t)(4 + 1 + 2 * (ach + bch + wch)) * 8192u;
        mbar_expect_tx(bar_tma, bytes);
        tma_load_4d(sm + OFF_QIN, &tm_q, bar_tma, 0, h, t0, bb);
        tma_load_4d(sm + OFF_QIN + 8192, &tm_q, bar_tma, 64, h, t0, bb);
        tma_load_4d(sm + OFF_KIN, &tm_k, bar_tma, 0, h, t0, bb);
        tma_load_4d(sm + OFF_KIN + 8192, &tm_k, bar_tma, 64, h, t0, bb);
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

    // ---- initial state: row `tid` of the slice, fp32 in registers ----------
    float S[NV];
    {
        const float* s0 = p.S0 ? p.S0 + (((size_t)bb * H + h) * DK + tid) * p.dv + v0 : nullptr;
#pragma unroll
        for (int j = 0; j < NV; j += 4) {
            float4 x = s0 ? *reinterpret_cast<const float4*>(s0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_SBF, sw128_chunk(tid, ch, DK), &S[8 * ch]);
    }
    if (tid == 0 && nchunks > 0) issue_loads(0);

#define GDR_WAIT(bar, ph)                                                   \
    do {                                                                    \
        bool w_ok = mbar_wait(bar, ph);                                     \
        ph ^= 1u;                                                           \
        if (!__syncthreads_and(w_ok)) { ok = false; goto finish; }          \
    } while (0)

    for (int ci = 0; ci < nchunks; ++ci) {
        const int t0 = ci * C;
        const int n = min(C, T - t0);
        // ---- scalar gates of this chunk (plain loads) ----------------------
        if (tid < C) {
            const int t = t0 + tid;
            const bool valid = t < T;
            const size_t gi = ((size_t)bb * T + t) * H + h;
            const __nv_bfloat16* ap = (const __nv_bfloat16*)p.alpha;
            const __nv_bfloat16* bp = (const __nv_bfloat16*)p.bg;
            const __nv_bfloat16* wp = (const __nv_bfloat16*)p.wg;
            s_ascal[tid] = (p.akind == GDR_GATE_SCALAR && valid) ? __bfloat162float(ap[gi]) : 1.f;
            s_bscal[tid] = (p.bkind == GDR_GATE_SCALAR && valid) ? __bfloat162float(bp[gi])
                           : (p.bkind == GDR_GATE_NONE ? 0.f : 0.f);
            s_wscal[tid] = (p.wkind == GDR_GATE_SCALAR && valid) ? __bfloat162float(wp[gi])
                           : (p.wkind == GDR_GATE_NONE ? 1.f : 0.f);
        }
        GDR_WAIT(bar_tma, ph_tma);

        // ---- build: log-decay scan and scaled operands --------------------
        // thread = (channel group cg of 8 channels, token group rg of 8 tokens)
        {
            const int cg = tid & 15, rg = tid >> 4;
            const int ch0 = cg * 8;
            float lg[8][8];  // [token i][channel e]: log2 alpha, then inclusive prefix
            float loc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) loc[e] = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = rg * 8 + i;
                float a8[8];
                if (ach) {
                    ld_chunk(sm + OFF_GA, sw128_chunk(r, cg, C), a8);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) a8[e] = s_ascal[r];
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float la = (r < n) ? lg2_approx(a8[e]) : 0.f;
                    loc[e] += la;
                    lg[i][e] = loc[e];
                }
            }
            float* scan = reinterpret_cast<float*>(sm + OFF_SCAN);  // [8 rg][128 ch] totals
#pragma unroll
            for (int e = 0; e < 8; ++e) scan[rg * 128 + ch0 + e] = loc[e];
            __syncthreads();
            float pre[8], tot[8], l0[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) { pre[e] = 0.f; tot[e] = 0.f; }
#pragma unroll
            for (int g = 0; g < 8; ++g) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float x = scan[g * 128 + ch0 + e];
                    if (g < rg) pre[e] += x;
                    tot[e] += x;
                }
            }
            // l_0 = log2 alpha_0 = first token's value (token group 0's first entry)
            __syncthreads();
            if (rg == 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) scan[1024 + ch0 + e] = lg[0][e];
            }
            __syncthreads();
#pragma unroll
            for (int e = 0; e < 8; ++e) l0[e] = scan[1024 + ch0 + e];
            float ref[8];
            bool bad = false;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                ref[e] = 0.5f * (l0[e] + tot[e]);  // tot = l_{n-1} (padding adds 0)
                bad |= (l0[e] - tot[e]) > 230.f;
            }
            if (bad) flag_status(p.d_status, GDR_DEVICE_DECAY_RANGE);
            if (rg == 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    s_gC[ch0 + e] = ex2_approx(tot[e]);
                    s_fS[ch0 + e] = ex2_approx(tot[e] - ref[e]);
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = rg * 8 + i;
                float k8[8], q8[8], b8[8], w8[8];
                ld_chunk(sm + OFF_KIN, sw128_chunk(r, cg, C), k8);
                ld_chunk(sm + OFF_QIN, sw128_chunk(r, cg, C), q8);
                if (bch) ld_chunk(sm + OFF_GB, sw128_chunk(r, cg, C), b8);
                else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) b8[e] = s_bscal[r];
                }
                if (!TIED) {
                    if (p.wkind == GDR_GATE_TIED) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) w8[e] = b8[e];
                    } else if (wch) {
                        ld_chunk(sm + OFF_GW, sw128_chunk(r, cg, C), w8);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) w8[e] = s_wscal[r];
                    }
                }
                float rop_k[8], rop_q[8], rg_k[8], rg_q[8], cop_k[8], cop_w[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float l = lg[i][e] + pre[e];
                    const float rowf = ex2_approx(l - ref[e]);
                    const float colf = ex2_approx(ref[e] - l);
                    const float g = ex2_approx(l);
                    const float kk = (r < n) ? k8[e] : 0.f;
                    const float qq = (r < n) ? q8[e] : 0.f;
                    rop_k[e] = b8[e] * kk * rowf;
                    rop_q[e] = qq * rowf;
                    rg_k[e] = b8[e] * kk * g;
                    rg_q[e] = qq * g;
                    cop_k[e] = kk * colf;
                    cop_w[e] = TIED ? 0.f : w8[e] * kk * colf;
                }
                st_chunk(sm + OFF_ROP, sw128_chunk(r, cg, 128), rop_k);
                st_chunk(sm + OFF_ROP, sw128_chunk(64 + r, cg, 128), rop_q);
                st_chunk(sm + OFF_RG, sw128_chunk(r, cg, 128), rg_k);
                st_chunk(sm + OFF_RG, sw128_chunk(64 + r, cg, 128), rg_q);
                st_chunk(sm + OFF_COP, sw128_chunk(r, cg, N1), cop_k);
                if (!TIED) st_chunk(sm + OFF_COP, sw128_chunk(64 + r, cg, N1), cop_w);
            }
        }
        __syncthreads();  // scan scratch (over X) is dead from here on
        if (TIED) {
            // X = [-Diag(beta) ; 0]: row t, 8 chunks of 8 columns
            float z[8];
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    z[e] = (tid < 64 && c8 * 8 + e == tid) ? -s_bscal[tid] : 0.f;
                st_chunk(sm + OFF_X, sw128_chunk(tid, c8, 128), z);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- P1: D1 = Rop x Cop^T ------------------------------------------
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

        // ---- unload D1: A (fp32), [0 ; -Aq] (bf16), X for general gates ------
        {
            const int r = tid & 63;
            float d[64];
            tmem_ld32(tmem + lane_base + TM_D1, d);
            tmem_ld32(tmem + lane_base + TM_D1 + 32, d + 32);
            if (tid < 64) {
                float* A32 = reinterpret_cast<float*>(sm + OFF_A32);
#pragma unroll
                for (int j = 0; j < 64; j += 4) {
                    float4 x = make_float4(j < r ? d[j] : 0.f, j + 1 < r ? d[j + 1] : 0.f,
                                           j + 2 < r ? d[j + 2] : 0.f, j + 3 < r ? d[j + 3] : 0.f);
                    *reinterpret_cast<float4*>(f32_at(A32, r, j)) = x;
                }
                float z[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) z[e] = 0.f;
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) st_chunk(sm + OFF_AP, sw128_chunk(tid, c8, 128), z);
            } else {
                float x[8];
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = c8 * 8 + e;
                        x[e] = j <= r ? -d[j] : 0.f;
                    }
                    st_chunk(sm + OFF_AP, sw128_chunk(tid, c8, 128), x);
                }
            }
            if (!TIED) {
                tmem_ld32(tmem + lane_base + TM_D1 + 64, d);
                tmem_ld32(tmem + lane_base + TM_D1 + 96, d + 32);
                float x[8];
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = c8 * 8 + e;
                        x[e] = (tid < 64 ? j < r : j <= r) ? d[j] : 0.f;
                    }
                    st_chunk(sm + OFF_X, sw128_chunk(tid, c8, 128), x);
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- solve T = (I + A)^-1, 16x16 blocks -------------------------------
        {
            float* A32 = reinterpret_cast<float*>(sm + OFF_A32);
            float* T32 = reinterpret_cast<float*>(sm + OFF_T32);
            float* P32 = reinterpret_cast<float*>(sm + OFF_P32);
            if (tid < 64) {
                // diagonal block I, column c: forward substitution
                const int I = tid >> 4, c = tid & 15;
                float x[16];
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) {
                    float s = (rr == c) ? 1.f : 0.f;
#pragma unroll
                    for (int j = 0; j < rr; ++j) s -= *f32_at(A32, 16 * I + rr, 16 * I + j) * x[j];
                    x[rr] = s;
                }
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) *f32_at(T32, 16 * I + rr, 16 * I + c) = x[rr];
            } else {
                // zero the strictly upper blocks of T (rows 0..47)
                const int u = tid - 64;  // 64 threads
                for (int idx = u; idx < 6 * 256; idx += 64) {
                    const int blk = idx >> 8, e = idx & 255;
                    // upper blocks (I,J) with J > I: (0,1)(0,2)(0,3)(1,2)(1,3)(2,3)
                    const int I = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
                    const int J = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
                    *f32_at(T32, 16 * I + (e >> 4), 16 * J + (e & 15)) = 0.f;
                }
            }
            __syncthreads();
            for (int dlev = 1; dlev <= 3; ++dlev) {
                const int nb = 4 - dlev;
                // stage a: P_IJ = sum_{K=J}^{I-1} A_IK T_KJ, units of 2 rows x 4 cols
                for (int u = tid; u < nb * 32; u += NT) {
                    const int bi = u >> 5, rr = ((u >> 2) & 7) * 2, c4 = (u & 3) * 4;
                    const int I = dlev + bi, J = bi;
                    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
                    for (int K = J; K < I; ++K) {
#pragma unroll
                        for (int m = 0; m < 16; ++m) {
                            const float a0 = *f32_at(A32, 16 * I + rr, 16 * K + m);
                            const float a1 = *f32_at(A32, 16 * I + rr + 1, 16 * K + m);
                            const float4 t4 = *reinterpret_cast<const float4*>(f32_at(T32, 16 * K + m, 16 * J + c4));
                            acc0[0] += a0 * t4.x; acc0[1] += a0 * t4.y; acc0[2] += a0 * t4.z; acc0[3] += a0 * t4.w;
                            acc1[0] += a1 * t4.x; acc1[1] += a1 * t4.y; acc1[2] += a1 * t4.z; acc1[3] += a1 * t4.w;
                        }
                    }
                    float* pb = P32 + bi * 256;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        pb[rr * 16 + c4 + e] = acc0[e];
                        pb[(rr + 1) * 16 + c4 + e] = acc1[e];
                    }
                }
                __syncthreads();
                // stage b: T_IJ = -T_II P_IJ
                for (int u = tid; u < nb * 32; u += NT) {
                    const int bi = u >> 5, rr = ((u >> 2) & 7) * 2, c4 = (u & 3) * 4;
                    const int I = dlev + bi, J = bi;
                    const float* pb = P32 + bi * 256;
                    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float t0v = *f32_at(T32, 16 * I + rr, 16 * I + m);
                        const float t1v = *f32_at(T32, 16 * I + rr + 1, 16 * I + m);
                        const float4 p4 = *reinterpret_cast<const float4*>(pb + m * 16 + c4);
                        acc0[0] += t0v * p4.x; acc0[1] += t0v * p4.y; acc0[2] += t0v * p4.z; acc0[3] += t0v * p4.w;
                        acc1[0] += t1v * p4.x; acc1[1] += t1v * p4.y; acc1[2] += t1v * p4.z; acc1[3] += t1v * p4.w;
                    }
                    *reinterpret_cast<float4*>(f32_at(T32, 16 * I + rr, 16 * J + c4)) =
                        make_float4(-acc0[0], -acc0[1], -acc0[2], -acc0[3]);
                    *reinterpret_cast<float4*>(f32_at(T32, 16 * I + rr + 1, 16 * J + c4)) =
                        make_float4(-acc1[0], -acc1[1], -acc1[2], -acc1[3]);
                }
                __syncthreads();
            }
            // L = [[T, 0], [0, I]] as bf16 [128 x 128]: thread = row
            {
                float x[8];
#pragma unroll
                for (int c8 = 0; c8 < 16; ++c8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = c8 * 8 + e;
                        if (tid < 64) x[e] = j < 64 ? *f32_at(T32, tid, j) : 0.f;
                        else x[e] = (j == tid) ? 1.f : 0.f;
                    }
                    st_chunk(sm + OFF_L, sw128_chunk(tid, c8, 128), x);
                }
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- P2: D2 = L x [Rg | X] -------------------------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idA = idesc_bf16(128, 128, 0, 1);
            const uint32_t idX = idesc_bf16(128, 64, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t ad = sdesc_sw128(sbase + OFF_L + (ks >> 2) * 16384u + (ks & 3) * 32u, 16, 1024);
                mma_bf16(tmem + TM_D2, ad, sdesc_sw128(sbase + OFF_RG + ks * 2048u, 16384, 1024), idA, ks > 0);
                mma_bf16(tmem + TM_D2 + 128, ad, sdesc_sw128(sbase + OFF_X + ks * 2048u, 16384, 1024), idX, ks > 0);
            }
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();

        // next chunk's inputs may now overwrite the input region (A32, T32, L
        // were last read above / by P2) -- except AP, read by P3 below.
        // ---- E_top = D2 rows 0..63 -> bf16 ----------------------------------
        if (tid < 64) {
            float d[32];
#pragma unroll
            for (int cb = 0; cb < 6; ++cb) {
                tmem_ld32(tmem + lane_base + TM_D2 + cb * 32, d);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) st_chunk(sm + OFF_E, sw128_chunk(tid, cb * 4 + c4, 128), d + 8 * c4);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- P3: D2 += [0 ; -Aq] x E_top --------------------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 192, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + TM_D2, sdesc_sw128(sbase + OFF_AP + ks * 32u, 16, 1024),
                         sdesc_sw128(sbase + OFF_E + ks * 2048u, 16384, 1024), id, 1);
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        if (tid == 0 && ci + 1 < nchunks) {
            fence_proxy_async();
            issue_loads(ci + 1);
        }

        // ---- E_bot = D2 rows 64..127 -> bf16 ----------------------------------
        if (tid >= 64) {
            float d[32];
#pragma unroll
            for (int cb = 0; cb < 6; ++cb) {
                tmem_ld32(tmem + lane_base + TM_D2 + cb * 32, d);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) st_chunk(sm + OFF_E, sw128_chunk(tid, cb * 4 + c4, 128), d + 8 * c4);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- S1: D3 = E x [S ; V] ---------------------------------------------
        const uint32_t vbuf = sbase + OFF_V + (ci & 1) * 8192u;
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, NV, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 12; ++ks) {
                const uint64_t ad = sdesc_sw128(sbase + OFF_E + (ks >> 2) * 16384u + (ks & 3) * 32u, 16, 1024);
                const uint64_t bd = ks < 8 ? sdesc_sw128(sbase + OFF_SBF + ks * 2048u, 8192, 1024)
                                           : sdesc_sw128(vbuf + (ks - 8) * 2048u, 8192, 1024);
                mma_bf16(tmem + TM_D3, ad, bd, id, ks > 0);
            }
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();

        // ---- epilogue: U -> smem, O -> global -----------------------------------
        {
            float d[64];
            tmem_ld32(tmem + lane_base + TM_D3, d);
            tmem_ld32(tmem + lane_base + TM_D3 + 32, d + 32);
            if (tid < 64) {
                float x[8];
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = -d[c8 * 8 + e];
                    st_chunk(sm + OFF_U, sw128_chunk(tid, c8, 64), x);
                }
            } else {
                const int t = t0 + tid - 64;
                if (t < T) {
                    __nv_bfloat16* op = p.o + (((size_t)bb * T + t) * H + h) * p.dv + v0;
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8) {
                        uint4 u;
                        u.x = pack_bf16x2(d[c8 * 8 + 0], d[c8 * 8 + 1]);
                        u.y = pack_bf16x2(d[c8 * 8 + 2], d[c8 * 8 + 3]);
                        u.z = pack_bf16x2(d[c8 * 8 + 4], d[c8 * 8 + 5]);
                        u.w = pack_bf16x2(d[c8 * 8 + 6], d[c8 * 8 + 7]);
                        *reinterpret_cast<uint4*>(op + c8 * 8) = u;
                    }
                }
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- S2: D4 = Cop^T x [U ; V] ------------------------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, NV, 1, 1);
#pragma unroll
            for (int ks = 0; ks < N1 / 16; ++ks) {
                const uint64_t ad = sdesc_sw128(sbase + OFF_COP + ks * 2048u, N1 * 128, 1024);
                const uint64_t bd = ks < 4 ? sdesc_sw128(sbase + OFF_U + ks * 2048u, 8192, 1024)
                                           : sdesc_sw128(vbuf + (ks - 4) * 2048u, 8192, 1024);
                mma_bf16(tmem + TM_D4, ad, bd, id, ks > 0);
            }
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();

        // ---- state update: S = Diag(g) S + Diag(f) D4 ------------------------
        {
            float d[64];
            tmem_ld32(tmem + lane_base + TM_D4, d);
            tmem_ld32(tmem + lane_base + TM_D4 + 32, d + 32);
            const float gC = s_gC[tid], fS = s_fS[tid];
#pragma unroll
            for (int j = 0; j < NV; ++j) S[j] = gC * S[j] + fS * d[j];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_SBF, sw128_chunk(tid, ch, DK), &S[8 * ch]);
        }
        tc_fence_before();
        __syncthreads();
    }

    if (p.ST) {
        float* st = p.ST + (((size_t)bb * H + h) * DK + tid) * p.dv + v0;
#pragma unroll
        for (int j = 0; j < NV; j += 4) *reinterpret_cast<float4*>(st + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }

finish:
    if (!ok && tid == 0) flag_status(p.d_status, GDR_DEVICE_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
#undef GDR_WAIT
}

}  // namespace chunk

// Host-side launch (tensor maps are built by the caller).
cudaError_t launch_chunk_sm100(const CUtensorMap* maps, const void* alpha, const void* b,
                               const void* w, int akind, int bkind, int wkind, bool tied,
                               const float* S0, void* o, float* ST, int* d_status, int B, int T,
                               int H, int dv, cudaStream_t st) {
    chunk::Params p;
    p.alpha = alpha; p.bg = b; p.wg = w;
    p.S0 = S0; p.o = (__nv_bfloat16*)o; p.ST = ST; p.d_status = d_status;
    p.B = B; p.T = T; p.H = H; p.dv = dv;
    p.akind = akind; p.bkind = bkind; p.wkind = wkind;
    dim3 grid(dv / chunk::NV, H, B);
    cudaError_t e;
    if (tied) {
        e = cudaFuncSetAttribute(chunk::chunk_fwd_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, chunk::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        chunk::chunk_fwd_kernel<true><<<grid, chunk::NT, chunk::SMEM_BYTES, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], p);
    } else {
        e = cudaFuncSetAttribute(chunk::chunk_fwd_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, chunk::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        chunk::chunk_fwd_kernel<false><<<grid, chunk::NT, chunk::SMEM_BYTES, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], p);
    }
    return cudaGetLastError();
}

}  // namespace gdr
