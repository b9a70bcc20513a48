// Chunkwise pass of the state gradient for the Gated DeltaNet form (scalar
// decay per token, tied scalar b = w = beta, d_k = d_v = 128, bf16 inputs) on
// sm_100a tensor cores: the backward pass's only sequential part.
//
// The state gradient G_t = dL/dS_t obeys G_t = q_t^T dO_t + M_{t+1} G_{t+1}
// with M_t = alpha_t (I - beta_t k_t^T k_t) (the transposed transition of the
// recurrence; symmetric for this gate form), and the token gradients that
// need it are dv_t = beta_t k_t G_t and dr_t = -k_t G_t (r_t the erase read).
// Over one chunk (tokens j = 0..n-1, g_j the decay product from the chunk's
// start, A and T = (I + A)^-1 the forward's masked key products and their UT
// transform, Aq the forward's masked, decay-scaled q k^T block), with G_in the
// gradient that later tokens (or dS_T) send into the chunk's last state and
// Y_j = k_j G_j, the reverse recurrence solves in closed form:
//   (I + A)^T Y = Diag(g_{n-1}/g) K G_in + Aq^T dO
//   G_out       = g_{n-1} G_in + (Diag(g) Q)^T dO - (Diag(beta g) K)^T Y
// (the chunk form of the forward transposed: the same triangular system,
// solved from the other side), and G_out flows into the previous chunk.
// Written as products on tensor cores:
//   pass 1 (every (chunk, head) item at once):
//     X   = (Diag(g_{n-1}/g) T)^T K          -> workspace [B,T,H,128]
//     AqT = Aq T                              -> workspace [B,T,H,64]
//     Q~  = Diag(g) Q                         -> workspace [B,T,H,128]
//   pass 2 (one CTA per (batch, head, 64 columns of d_v), chunks in reverse):
//     Y     = AqT^T dO + X G_in               (dv = beta Y, dr = -Y per token)
//     G_out = g_{n-1} G_in + Q~^T dO + K^T (-beta g Y)
// The per-chunk chain is the forward state pass's: one product over d_k
// (X G_in), one over the chunk's tokens (K^T Y'), with the dO products off the
// chain. The reverse-mode derivative of the recurrence is the gate-aware
// backward of "Erase-then-Delta Attention" (abstract); its chunk form is
// checked against the oracle's reverse token loop.
#include "chunk_common.cuh"

namespace gdr {
namespace bwdgrad {

using namespace chunkc;

// ---- pass 1 shared memory (bytes from a 1024-aligned base) ----------------
constexpr uint32_t B_OFF_K = 0;         // K [64 x 128] bf16, two 8 KB column blocks; 2 buffers
constexpr uint32_t B_OFF_Q = 32768;     // Q (one buffer); scaled in place to Diag(g) Q and stored
constexpr uint32_t B_OFF_AQ = 49152;    // Aq bf16 [64 x 64] (A operand of Aq T)
constexpr uint32_t B_OFF_A32 = 57344;   // A fp32; then Diag(g_{n-1}/g) T | T (bf16); then X staging
constexpr uint32_t B_OFF_T32 = 73728;   // T fp32 [64 x 64]; then AqT staging
constexpr uint32_t B_OFF_SCR = 90112;   // solve scratch fp32 (5 KB)
constexpr uint32_t B_OFF_SMALL = 95232;
constexpr uint32_t B_SMEM_BYTES = B_OFF_SMALL + 2048 + 1024;
// TMEM: K K^T (columns 0..63, lanes 0..63), Q K^T (columns 64..127, lanes
// 64..127); then AqT (columns 0..63) and X (columns 128..255), lanes 0..63.
constexpr uint32_t B_TM_D1 = 0, B_TM_DQ = 64, B_TM_AQT = 0, B_TM_X = 128, B_TM_COLS = 256;

struct PrepParams {
    const void* alpha;
    const void* beta;
    int* d_status;
    int T, H, nitems;
    int group;  // value heads per q/k head (q, k read at head h / group)
};

__global__ void __launch_bounds__(NT, 2) prep_grad_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                          const __grid_constant__ CUtensorMap tm_k,
                                                          const __grid_constant__ CUtensorMap tm_xout,
                                                          const __grid_constant__ CUtensorMap tm_aqtout,
                                                          const __grid_constant__ CUtensorMap tm_qtout,
                                                          const PrepParams pp) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, wg = warp >> 2, row = tid & 127;
    const int T = pp.T, H = pp.H;
    const int nchunks = (T + C - 1) / C;

    float* s_beta = reinterpret_cast<float*>(sm + B_OFF_SMALL);
    float* s_alpha = s_beta + 64;
    float* s_l = s_beta + 128;    // log2 prefix of alpha over the chunk
    float* s_g = s_beta + 192;    // 2^l
    float* s_gcr = s_beta + 256;  // 2^(l_{n-1} - l)
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + B_OFF_SMALL + 1280);  // [2]: K
    uint64_t* bar_mma = bar_tma + 2;
    uint64_t* bar_q = bar_tma + 3;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + B_OFF_SMALL + 1328);
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
        mbar_expect_tx(&bar_tma[buf], 2u * 8192u);
        tma_load_4d(sm + B_OFF_K + buf * 16384, &tm_k, &bar_tma[buf], 0, h / pp.group, ci * C, bb);
        tma_load_4d(sm + B_OFF_K + buf * 16384 + 8192, &tm_k, &bar_tma[buf], 64, h / pp.group, ci * C, bb);
    };
    auto issue_q = [&](int item) {
        int ci, h, bb;
        coords(item, ci, h, bb);
        mbar_expect_tx(bar_q, 2u * 8192u);
        tma_load_4d(sm + B_OFF_Q, &tm_q, bar_q, 0, h / pp.group, ci * C, bb);
        tma_load_4d(sm + B_OFF_Q + 8192, &tm_q, bar_q, 64, h / pp.group, ci * C, bb);
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

    // the gradient state pass may be scheduled now; it waits for this grid's
    // completion before its first workspace read
    asm volatile("griddepcontrol.launch_dependents;");
    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_q, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_xout);
        prefetch_tmap(&tm_aqtout);
        prefetch_tmap(&tm_qtout);
        if ((int)blockIdx.x < pp.nitems) {
            issue_k(blockIdx.x, 0);
            issue_q(blockIdx.x);
        }
    }
    if ((int)blockIdx.x < pp.nitems) load_gates(blockIdx.x);
    if (warp == 0) tmem_alloc(s_tmem, B_TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t ph_tma0 = 0, ph_tma1 = 0, ph_mma = 0, ph_q = 0;
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
        const uint32_t kb = sbase + B_OFF_K + buf * 16384u;
        if (tid < C) {
            const bool valid = tid < n;
            s_alpha[tid] = valid ? bits_to_f32(g_a) : 1.f;
            s_beta[tid] = valid ? bits_to_f32(g_b) : 0.f;
        }
        // the next item's K: its buffer was last read by this CTA's previous X product
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
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t koff = (ks >> 2) * 8192u + (ks & 3) * 32u;
                mma_bf16(tmem + B_TM_D1, sdesc_sw128(kb + koff, 16, 1024), sdesc_sw128(kb + koff, 16, 1024),
                         id, ks > 0);
                mma_bf16(tmem + B_TM_DQ, sdesc_sw128(sbase + B_OFF_Q - 8192 + koff, 16, 1024),
                         sdesc_sw128(kb + koff, 16, 1024), id, ks > 0);
            }
            mma_commit(bar_mma);
            // the previous item's stores (X and AqT out of the A32 / T32 tiles)
            // have read them before A and T are written again
            bulk_wait_group_read0();
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();

        if ((warp & 3) < 2) {
            // ---- A (fp32, strict lower) and its transposed 16 x 16 diagonal blocks ----
            const int r = row;  // 0..63
            float d[32];
            tmem_ld32(tmem + lane_base + B_TM_D1 + wg * 32, d);
            const float rf = s_beta[r], lr = s_l[r];
            float* A32 = reinterpret_cast<float*>(sm + B_OFF_A32);
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
                float* at = reinterpret_cast<float*>(sm + B_OFF_SCR) + I * 272;
                if (I & 1) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) at[j * 16 + rr] = d[16 + j];
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) at[j * 16 + rr] = d[j];
                }
            }
        } else {
            // ---- Aq_tj = (q_t . k_j) 2^(l_t - l_j), j <= t (bf16), then Q~ = Diag(g) Q ----
            const int t = row - 64;
            float d[32];
            tmem_ld32(tmem + lane_base + B_TM_DQ + wg * 32, d);
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
                st_chunk(sm + B_OFF_AQ, sw128_chunk(t, wg * 4 + c8, 64), x);
            }
            // Q~ in place (Q K^T has read Q): 1024 16-byte pieces of two 64 x 64
            // blocks, a piece's row is its 128-byte line within its block
            const int uu = wg ? tid - 128 : tid - 64;  // 0..127 over warps 2, 3, 6, 7
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t off = (uint32_t)(uu + 128 * i) * 16u;
                const float f = s_g[(off & 8191u) >> 7];
                float x[8];
                ld_chunk(sm + B_OFF_Q, off, x);
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] *= f;
                st_chunk(sm + B_OFF_Q, off, x);
            }
        }
        fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&tm_qtout, sm + B_OFF_Q, 0, h, t0, bb);
            tma_store_4d(&tm_qtout, sm + B_OFF_Q + 8192, 64, h, t0, bb);
            bulk_commit_group();
        }

        // ---- T = (I + A)^-1; Diag(g_{n-1}/g) T and T in bf16 ------------------------
        {
            float* A32 = reinterpret_cast<float*>(sm + B_OFF_A32);
            float* T32 = reinterpret_cast<float*>(sm + B_OFF_T32);
            solve_unit_lower(A32, T32, reinterpret_cast<float*>(sm + B_OFF_SCR), tid, warp);
            const int r = tid & 63, q4 = tid >> 6;
            const float fr = s_gcr[r];
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
                    y[e4] = t4.x; y[e4 + 1] = t4.y; y[e4 + 2] = t4.z; y[e4 + 3] = t4.w;
                    x[e4] = fr * t4.x; x[e4 + 1] = fr * t4.y; x[e4 + 2] = fr * t4.z; x[e4 + 3] = fr * t4.w;
                }
                st_chunk(sm + B_OFF_A32, sw128_chunk(r, c8, 64), x);         // Diag(g_{n-1}/g) T
                st_chunk(sm + B_OFF_A32 + 8192, sw128_chunk(r, c8, 64), y);  // T
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- X = (Diag(g_{n-1}/g) T)^T K (N = 128), AqT = Aq T (N = 64) -------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idX = idesc_bf16(128, 128, 1, 1);
            const uint32_t idA = idesc_bf16(128, 64, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                // A = (Diag(g_{n-1}/g) T)^T: MN-major over the [m][j] tile; its second
                // 64-row block (rows 64..127 of the M = 128 operand) is the T tile: garbage rows
                mma_bf16(tmem + B_TM_X, sdesc_sw128(sbase + B_OFF_A32 + ks * 2048u, 8192, 1024),
                         sdesc_sw128(kb + ks * 2048u, 8192, 1024), idX, ks > 0);
                mma_bf16(tmem + B_TM_AQT, sdesc_sw128(sbase + B_OFF_AQ + ks * 32u, 16, 1024),
                         sdesc_sw128(sbase + B_OFF_A32 + 8192 + ks * 2048u, 8192, 1024), idA, ks > 0);
            }
            mma_commit(bar_mma);
        }
        GDR_WAIT(bar_mma, ph_mma);
        tc_fence_after();
        if (tid == 0 && next < pp.nitems) {
            bulk_wait_group_read0();  // the Q~ store has left the Q tile
            issue_q(next);
        }

        // ---- X -> staging over A32, AqT -> staging over T32 (rows 0..63) -------------
        if ((warp & 3) < 2) {
            const int r = row;
            float d[32], d1[32];
            tmem_ld32_async(tmem + lane_base + B_TM_X + wg * 64, d);
            tmem_ld32_async(tmem + lane_base + B_TM_X + wg * 64 + 32, d1);
            tmem_wait_ld();
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8)
                st_chunk(sm + B_OFF_A32, sw128_chunk(r, wg * 8 + c8, 64), c8 < 4 ? d + c8 * 8 : d1 + (c8 - 4) * 8);
            tmem_ld32(tmem + lane_base + B_TM_AQT + wg * 32, d);
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) st_chunk(sm + B_OFF_T32, sw128_chunk(r, wg * 4 + c8, 64), d + c8 * 8);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&tm_xout, sm + B_OFF_A32, 0, h, t0, bb);
            tma_store_4d(&tm_xout, sm + B_OFF_A32 + 8192, 64, h, t0, bb);
            tma_store_4d(&tm_aqtout, sm + B_OFF_T32, 0, h, t0, bb);
            bulk_commit_group();
        }
    }

finish:
    if (!ok && tid == 0) flag_status(pp.d_status, GDR_DEVICE_TIMEOUT);
    if (tid == 0) bulk_wait_group0();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, B_TM_COLS);
#undef GDR_WAIT
}

// ---- pass 2 shared memory ---------------------------------------------------
// Inputs triple-buffered (step n + 2 loads while step n runs). The M = 128
// operands read 64 garbage rows past each 64-row tile: X's second block and
// then AqT, AqT's next 8 KB (Q~).
constexpr int G_NBUF = 3;
constexpr uint32_t G_STAGE = 65536;
constexpr uint32_t G_ST_X = 0;        // X [64 x 128] bf16 (K-major A of X G)
constexpr uint32_t G_ST_AQT = 16384;  // AqT [64 x 64] (MN-major A of AqT^T dO)
constexpr uint32_t G_ST_QT = 24576;   // Q~ [64 x 128] (MN-major A of Q~^T dO)
constexpr uint32_t G_ST_K = 40960;    // K [64 x 128] (MN-major A of K^T Y')
constexpr uint32_t G_ST_DO = 57344;   // dO slice [64 x 64] (MN-major B)
constexpr uint32_t G_OFF_SBF = G_NBUF * G_STAGE;  // G bf16 [128 x 64] (B operand, MN-major)
constexpr uint32_t G_OFF_Y = G_OFF_SBF + 16384;   // Y' = -Diag(beta g) Y bf16 [64 x 64]
constexpr uint32_t G_OFF_SMALL = G_OFF_Y + 8192;
constexpr uint32_t G_SMEM_BYTES = G_OFF_SMALL + 2048 + 1024;
// TMEM: Y (lanes 0..63) and the G_out increment, each in two column sets by
// step parity so a step's dO products can be issued before the previous step ends
constexpr uint32_t G_TM_Y = 0, G_TM_G = 128, G_TM_COLS = 256;
constexpr int G_NT = 288;  // warps 0..7 compute, warp 8 issues every MMA and TMA load
constexpr int G_BAR_STEP = 1;

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

struct GradParams {
    const void* alpha;  // [B, T, H] scalar gates (bf16)
    const void* beta;
    const float* dST;   // [B, H, 128, d_v] or NULL
    __nv_bfloat16* ckG; // [B, H, nchunks, 128, d_v] bf16: G_in of every chunk
    __nv_bfloat16* DR;  // [B, T, H, d_v] bf16: dr = -k G
    float* dv;          // [B, T, H, d_v]: beta k G
    float* dS0;         // [B, H, 128, d_v] or NULL
    int* d_status;
    int T, H, dv_;
    int group;
};

// Step n of a CTA handles chunk ci = nchunks - 1 - n. The issuer issues the
// step's two dO products as soon as its tiles land, X G once the state copy of
// the previous step is written (s_ready), K^T Y' once Y' is (y_ready).
__global__ void __launch_bounds__(G_NT, 1) state_grad_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_aqt,
    const __grid_constant__ CUtensorMap tm_qt, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_do, const GradParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = (warp >> 2) & 1;
    const int row = tid & 127;  // TMEM lane / state row (compute threads)
    const bool lo = row < 64;   // warps 0, 1, 4, 5: lanes 0..63 (token rows of Y)
    const int vt = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int hq = h / p.group;
    const int v0 = vt * NV;
    const int T = p.T, H = p.H;
    const int nchunks = (T + C - 1) / C;

    // per-step factors, three sets by step % 3 (written one step ahead):
    // beta, beta g (g = 2^l, l the log2 prefix of alpha over the chunk), g_{n-1}
    float* s_b3 = reinterpret_cast<float*>(sm + G_OFF_SMALL);  // [3][64]
    float* s_bg3 = s_b3 + 192;                                 // [3][64]
    float* s_gC3 = s_b3 + 384;                                 // [3][4]
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + G_OFF_SMALL + 1600);  // [3]
    uint64_t* bar_w = bar_tma + 3;    // Y complete
    uint64_t* bar_k = bar_tma + 4;    // G_out increment complete
    uint64_t* bar_drain = bar_tma + 5;
    uint64_t* y_ready = bar_tma + 6;  // Y' written (compute -> issuer)
    uint64_t* s_ready = bar_tma + 7;  // state copy written
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + G_OFF_SMALL + 1664);
    if (tid == 0) {
        for (int i = 0; i < G_NBUF; ++i) mbar_init(&bar_tma[i], 1);
        mbar_init(bar_w, 1);
        mbar_init(bar_k, 1);
        mbar_init(bar_drain, 1);
        mbar_init(y_ready, 128);
        mbar_init(s_ready, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_aqt);
        prefetch_tmap(&tm_qt);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_do);
    }
    if (warp == 0) tmem_alloc(s_tmem, G_TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t sbase = smem_u32(sm);
    bool ok = true;

    constexpr int NH = NV / 2;
    float G[NH];  // state gradient: row `row`, columns v0 + 32 wg ..
    if (warp < 8) {
        const float* g0 = p.dST ? p.dST + (((size_t)bb * H + h) * DK + row) * p.dv_ + v0 + wg * NH : nullptr;
#pragma unroll
        for (int j = 0; j < NH; j += 4) {
            float4 x = g0 ? *reinterpret_cast<const float4*>(g0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            G[j] = x.x; G[j + 1] = x.y; G[j + 2] = x.z; G[j + 3] = x.w;
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) st_chunk(sm + G_OFF_SBF, sw128_chunk(row, wg * 4 + ch, DK), &G[8 * ch]);
    }

    // gates of a chunk by warp 2 (two tokens per lane): factors set n % 3
    auto bits_to_f32 = [](unsigned short u) { return __uint_as_float((uint32_t)u << 16); };
    unsigned short a0 = 0x3F80, a1 = 0x3F80, b0 = 0, b1 = 0;  // of the next chunk to scan
    auto load_gates = [&](int ci) {
        const int t = ci * C + 2 * lane;
        const unsigned short* ap = (const unsigned short*)p.alpha;
        const unsigned short* bp = (const unsigned short*)p.beta;
        a0 = t < T ? ap[((size_t)bb * T + t) * H + h] : (unsigned short)0x3F80;
        a1 = t + 1 < T ? ap[((size_t)bb * T + t + 1) * H + h] : (unsigned short)0x3F80;
        b0 = t < T ? bp[((size_t)bb * T + t) * H + h] : (unsigned short)0;
        b1 = t + 1 < T ? bp[((size_t)bb * T + t + 1) * H + h] : (unsigned short)0;
    };
    auto scan_gates = [&](int n) {
        const int s3 = n % 3;
        const float la0 = lg2_approx(bits_to_f32(a0));
        const float la1 = lg2_approx(bits_to_f32(a1));
        float x = la0 + la1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        const float l1 = x, l0v = x - la1;
        const float last = __shfl_sync(0xffffffffu, l1, 31);
        const float bf0 = bits_to_f32(b0), bf1 = bits_to_f32(b1);
        s_b3[s3 * 64 + 2 * lane] = bf0;
        s_b3[s3 * 64 + 2 * lane + 1] = bf1;
        s_bg3[s3 * 64 + 2 * lane] = bf0 * ex2_approx(l0v);
        s_bg3[s3 * 64 + 2 * lane + 1] = bf1 * ex2_approx(l1);
        if (lane == 0) s_gC3[s3 * 4] = ex2_approx(last);
    };

    auto issue_loads = [&](int n) {
        const int ci = nchunks - 1 - n, t0 = ci * C, buf = n % G_NBUF;
        uint8_t* st = sm + buf * G_STAGE;
        mbar_expect_tx(&bar_tma[buf], 8u * 8192u);
        tma_load_4d(st + G_ST_X, &tm_x, &bar_tma[buf], 0, h, t0, bb);
        tma_load_4d(st + G_ST_X + 8192, &tm_x, &bar_tma[buf], 64, h, t0, bb);
        tma_load_4d(st + G_ST_AQT, &tm_aqt, &bar_tma[buf], 0, h, t0, bb);
        tma_load_4d(st + G_ST_QT, &tm_qt, &bar_tma[buf], 0, h, t0, bb);
        tma_load_4d(st + G_ST_QT + 8192, &tm_qt, &bar_tma[buf], 64, h, t0, bb);
        tma_load_4d(st + G_ST_K, &tm_k, &bar_tma[buf], 0, hq, t0, bb);
        tma_load_4d(st + G_ST_K + 8192, &tm_k, &bar_tma[buf], 64, hq, t0, bb);
        tma_load_4d(st + G_ST_DO, &tm_do, &bar_tma[buf], v0, h, t0, bb);
    };

    fence_proxy_async();  // the gradient's bf16 copy is read by the first MMA
    tc_fence_before();
    // everything above overlaps the first pass's tail; its outputs are read
    // only after it has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == 8 && lane == 0)
        for (int n = 0; n < 2 && n < nchunks; ++n) issue_loads(n);
    if (warp == 2 && nchunks > 0) {
        load_gates(nchunks - 1);
        scan_gates(0);
        if (nchunks > 1) load_gates(nchunks - 2);
    }
    __syncthreads();

    int loads_issued = min(2, nchunks);
    if (warp == 8) {
        // ---------------- issuer warp ------------------------------------------------
        bool iok = true;
        for (int n = 0; n < nchunks && iok; ++n) {
            const int buf = n % G_NBUF, par = n & 1;
            const uint32_t ph = (uint32_t)(n & 1);
            const uint32_t stb = sbase + buf * G_STAGE;
            const uint32_t dY = G_TM_Y + (uint32_t)par * 64u, dG = G_TM_G + (uint32_t)par * 64u;
            iok = __all_sync(0xffffffffu, mbar_wait(&bar_tma[buf], (uint32_t)((n / G_NBUF) & 1)) && iok);
            if (!iok) break;
            tc_fence_after();
            if (lane == 0) {
                // the step's dO products (their column sets were read two steps ago)
                const uint32_t idT = idesc_bf16(128, NV, 1, 1);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t bdo = sdesc_sw128(stb + G_ST_DO + ks * 2048u, 8192, 1024);
                    mma_bf16(tmem + dY, sdesc_sw128(stb + G_ST_AQT + ks * 2048u, 8192, 1024), bdo, idT, ks > 0);
                    mma_bf16(tmem + dG, sdesc_sw128(stb + G_ST_QT + ks * 2048u, 8192, 1024), bdo, idT, ks > 0);
                }
            }
            __syncwarp();
            if (n > 0) {
                iok = __all_sync(0xffffffffu, mbar_wait(s_ready, (uint32_t)((n - 1) & 1)) && iok);
                if (!iok) break;
                tc_fence_after();
            }
            if (lane == 0) {
                // Y += X G_in (over d_k)
                const uint32_t idX = idesc_bf16(128, NV, 0, 1);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t koff = (ks >> 2) * 8192u + (ks & 3) * 32u;
                    mma_bf16(tmem + dY, sdesc_sw128(stb + G_ST_X + koff, 16, 1024),
                             sdesc_sw128(sbase + G_OFF_SBF + ks * 2048u, 8192, 1024), idX, 1);
                }
                mma_commit(bar_w);
                // step n + 2's inputs go to the stage of step n - 1, whose products
                // all finished before its gradient update (s_ready above)
                if (n + 2 < nchunks) issue_loads(n + 2);
            }
            if (n + 2 < nchunks) loads_issued = n + 3;
            __syncwarp();
            iok = __all_sync(0xffffffffu, mbar_wait(y_ready, ph) && iok);
            if (!iok) break;
            tc_fence_after();
            if (lane == 0) {
                // G_out increment += K^T Y'
                const uint32_t idT = idesc_bf16(128, NV, 1, 1);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + dG, sdesc_sw128(stb + G_ST_K + ks * 2048u, 8192, 1024),
                             sdesc_sw128(sbase + G_OFF_Y + ks * 2048u, 8192, 1024), idT, 1);
                mma_commit(bar_k);
            }
            __syncwarp();
        }
        if (!iok) {
            ok = false;
            if (lane == 0) {
                // before the block leaves (each wait bounded): the requested input
                // copies have landed and the issued MMAs have finished
                for (int n = max(0, loads_issued - G_NBUF); n < loads_issued; ++n)
                    (void)mbar_wait(&bar_tma[n % G_NBUF], (uint32_t)((n / G_NBUF) & 1));
                mma_commit(bar_drain);
                (void)mbar_wait(bar_drain, 0);
            }
            __syncwarp();
        }
    } else {
        // ---------------- compute warps ----------------------------------------------
        bool w_ok = true;
        int n = 0;
        for (; n < nchunks; ++n) {
            const int ci = nchunks - 1 - n;
            const int par = n & 1, s3 = n % 3;
            const uint32_t ph = (uint32_t)(n & 1);
            // G_in of the chunk (the gradient its last state receives from later
            // tokens), written by each thread for its row off the chunk chain
            auto store_ck = [&]() {
                __nv_bfloat16* dst = p.ckG + ((((size_t)bb * H + h) * nchunks + ci) * DK + row) * p.dv_ + v0 + wg * NH;
#pragma unroll
                for (int jj = 0; jj < NH; jj += 8)
                    *reinterpret_cast<uint4*>(dst + jj) =
                        make_uint4(pack_bf16x2(G[jj], G[jj + 1]), pack_bf16x2(G[jj + 2], G[jj + 3]),
                                   pack_bf16x2(G[jj + 4], G[jj + 5]), pack_bf16x2(G[jj + 6], G[jj + 7]));
            };
            if (lo) {
                // ---- Y of the chunk's tokens: dv, dr, and Y' = -Diag(beta g) Y ----------
                w_ok = mbar_wait(bar_w, ph) && w_ok;
                tc_fence_after();
                const int j = row;
                const int t = ci * C + j;
                float d[32];
                tmem_ld32(tmem + lane_base + G_TM_Y + (uint32_t)par * 64u + wg * 32, d);
                const float bj = s_b3[s3 * 64 + j], bgj = s_bg3[s3 * 64 + j];
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = -bgj * d[c8 * 8 + e];
                    st_chunk(sm + G_OFF_Y, sw128_chunk(j, wg * 4 + c8, 64), x);
                }
                fence_proxy_async();
                tc_fence_before();
                mbar_arrive(y_ready);
                // the token gradients and the checkpoint leave after K^T Y' may start
                if (t < T) {
                    const size_t off = (((size_t)bb * T + t) * H + h) * p.dv_ + v0 + wg * 32;
#pragma unroll
                    for (int c4 = 0; c4 < 32; c4 += 4)
                        *reinterpret_cast<float4*>(p.dv + off + c4) =
                            make_float4(bj * d[c4], bj * d[c4 + 1], bj * d[c4 + 2], bj * d[c4 + 3]);
#pragma unroll
                    for (int c8 = 0; c8 < 32; c8 += 8)
                        *reinterpret_cast<uint4*>(p.DR + off + c8) =
                            make_uint4(pack_bf16x2(-d[c8], -d[c8 + 1]), pack_bf16x2(-d[c8 + 2], -d[c8 + 3]),
                                       pack_bf16x2(-d[c8 + 4], -d[c8 + 5]), pack_bf16x2(-d[c8 + 6], -d[c8 + 7]));
                }
                store_ck();
            } else {
                store_ck();
                if (warp == 2 && n + 1 < nchunks) {
                    scan_gates(n + 1);
                    if (n + 2 < nchunks) load_gates(ci - 2);
                }
            }
            // ---- G_out = g_{n-1} G_in + (Q~^T dO + K^T Y') -----------------------------
            w_ok = mbar_wait(bar_k, ph) && w_ok;
            tc_fence_after();
            {
                float dG[32];
                tmem_ld32(tmem + lane_base + G_TM_G + (uint32_t)par * 64u + wg * 32, dG);
                const float gC = s_gC3[s3 * 4];
#pragma unroll
                for (int jj = 0; jj < NH; ++jj) G[jj] = fmaf(gC, G[jj], dG[jj]);
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) st_chunk(sm + G_OFF_SBF, sw128_chunk(row, wg * 4 + ch, DK), &G[8 * ch]);
            }
            fence_proxy_async();  // the gradient copy feeds the next step's MMAs
            tc_fence_before();
            if (!named_bar_and(G_BAR_STEP, 256, w_ok)) break;
            if (tid == 0) mbar_arrive(s_ready);
        }
        if (n < nchunks) ok = false;  // a wait gave up
        if (ok && p.dS0) {
            float* dst = p.dS0 + (((size_t)bb * H + h) * DK + row) * p.dv_ + v0 + wg * NH;
#pragma unroll
            for (int jj = 0; jj < NH; jj += 4)
                *reinterpret_cast<float4*>(dst + jj) = make_float4(G[jj], G[jj + 1], G[jj + 2], G[jj + 3]);
        }
    }
    if (!ok && (tid == 0 || tid == 256)) flag_status(p.d_status, GDR_DEVICE_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, G_TM_COLS);
}

}  // namespace bwdgrad

// Workspace of the gradient pass's first pass, per token-head (bf16): X (128),
// AqT (64), Q~ (128).
size_t bwd_grad_workspace_bytes(int B, int T, int H) {
    return (size_t)B * T * H * (chunkc::DK + chunkc::C + chunkc::DK) * sizeof(__nv_bfloat16);
}

// maps: q, k ([B,T,H/group,128]) and dO ([B,T,H,128]); ws_maps: X ([B,T,H,128]),
// AqT ([B,T,H,64]), Q~ ([B,T,H,128]). Writes ckG and DR (bf16), dv and (if not
// NULL) dS0.
cudaError_t launch_bwd_grad_tc(const CUtensorMap* q_map, const CUtensorMap* k_map, const CUtensorMap* do_map,
                               const CUtensorMap* ws_maps, const void* alpha, const void* beta,
                               const float* dST, __nv_bfloat16* ckG, __nv_bfloat16* DR, float* dv, float* dS0,
                               int* d_status, int B, int T, int H, int dvn, int group, cudaStream_t st) {
    using namespace bwdgrad;
    if (dvn != 128) return cudaErrorInvalidValue;
    PrepParams pp;
    pp.alpha = alpha; pp.beta = beta;
    pp.d_status = d_status;
    pp.T = T; pp.H = H;
    pp.group = group;
    const int nchunks = (T + C - 1) / C;
    pp.nitems = nchunks * H * B;
    cudaError_t e = cudaFuncSetAttribute(prep_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, B_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int grid = min(pp.nitems, 2 * nsm);  // two resident CTAs per SM
    prep_grad_kernel<<<grid, NT, B_SMEM_BYTES, st>>>(*q_map, *k_map, ws_maps[0], ws_maps[1], ws_maps[2], pp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    GradParams gp;
    gp.alpha = alpha; gp.beta = beta; gp.dST = dST;
    gp.ckG = ckG; gp.DR = DR; gp.dv = dv; gp.dS0 = dS0;
    gp.d_status = d_status;
    gp.T = T; gp.H = H; gp.dv_ = dvn; gp.group = group;
    e = cudaFuncSetAttribute(state_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, G_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(dvn / NV, H, B);
    cfg.blockDim = dim3(G_NT, 1, 1);
    cfg.dynamicSmemBytes = G_SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap the first pass's tail
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, state_grad_kernel, ws_maps[0], ws_maps[1], ws_maps[2], *k_map, *do_map, gp);
}

}  // namespace gdr
