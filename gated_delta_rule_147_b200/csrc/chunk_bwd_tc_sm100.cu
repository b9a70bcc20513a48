// Chunk-parallel part of the backward pass on sm_100a tensor cores, for the
// Gated DeltaNet form (one decay per token, b = w = beta one scalar per token),
// bf16 inputs, d_k = d_v = 128.
//
// The gradients of a chunk follow from its start state S0, the state gradient
// G_e at its end and, per token, the erase read r_t and its gradient dr_t
// (checkpoints of the backward's forward and gradient passes, bf16; r comes as
// U = beta v - r): with r and dr known the
// chunk is a diagonal-decay system without erase, and every gradient is a
// masked product ("The Eraser Trilogy", "The Rosetta Stone": the masked-
// matrix form of such a system). With l_t the prefix sum of log2 alpha over
// the chunk, Gam_t = 2^l_t, G_tj = 2^(l_t - l_j) (t >= j), e = u = beta . k:
//   P1 = M  . G . (dO V^T),  P2 = M  . G . (dO R^T)    (M: j <= t)
//   P3 = M1 . G . (DR V^T),  P4 = M1 . G . (DR R^T)    (M1: j < t)
//   dq  = Gam . (dO S0^T) + P1 U - P2 K
//   de  = Gam . (DR S0^T) + P3 U - P4 K
//   du  = P1^T Q + P3^T E + (Gam_C / Gam) . (V G_e^T)
//   dkr = -(P2^T Q + P4^T E) - (Gam_C / Gam) . (R G_e^T)
//   dk  = dkr + beta (de + du),   dbeta = sum_c k . (de + du)
//   dalpha_s = dlam_s / alpha_s with dlam_s the derivative by log alpha_s.
//   A term of the chunk's output (or of its erase read) at token t that token
//   j wrote carries G_tj, which holds log alpha_s exactly for j < s <= t; the
//   start-state terms carry Gam_t (every s <= t); the end state's share
//   carries Gam_C / Gam_j (s > j) or Gam_C. Summing each term once:
//   dlam_s = sum_{t >= s} a_t + sum_{t >= s} sum_{j < s} M_tj
//            + Gam_C <G_e, S0> + sum_{j < s} c_j,
//   a_t  = Gam_t (q_t . (dO_t S0^T) + e_t . (dr_t S0^T)),
//   M_tj = (q_t . u_j) P1_tj - (q_t . k_j) P2_tj + (e_t . u_j) P3_tj - (e_t . k_j) P4_tj,
//   c_j  = u_j . du_j^G + k_j . dkr_j^G   (du^G, dkr^G: the G_e parts).
//   Forming dlam as the difference of q.dq and u.du would leave the j = t
//   terms (no decay) to cancel between two separately rounded sums.
// Every decay factor used is at most 1, so any alpha in (0, 1] is in range.
//
// One CTA per (chunk, head, batch), 256 threads; thread 0 loads every operand
// tile by TMA (q, k, v, dO, U, dr, S0, G_e) and issues the MMAs (bf16
// operands, fp32 accumulators in tensor memory), three products:
//   D12 = [dO ; DR] [S0 | V | Uf]^T           (N = 256: dO S0^T, DR S0^T and
//                                              the token-by-token blocks; Uf =
//                                              beta v - r is the forward's
//                                              checkpoint, so the R blocks are
//                                              beta_j (V block) - (Uf block))
//   D7  = [Q ; U] K^T                           (q_t . k_j and e_t . k_j for M)
//   D3  = [[P1, -P2] ; [P3, -P4]] [U ; K]       (dq and de without their S0 part)
//   D45 = [[P1, -P2] ; [P3, -P4]]^T [Q ; E]    (du', dkr')
//   D6  = [V' ; -R'] G_e^T                      (du^G, dkr^G)
// with V' = (Gam_C / Gam) . V and R' likewise.
#include "chunk_common.cuh"

namespace gdr {
namespace bwdtc {

using namespace chunkc;

// Named barrier `id` (1..15) over `n` threads (a multiple of 32): producers
// arrive, consumers wait.
__device__ __forceinline__ void named_bar_arrive(uint32_t id, uint32_t n) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

struct TcParams {
    const __nv_bfloat16 *alpha, *beta;     // scalar gates [B, T, H]
    float *dq, *dk, *dalpha, *db;          // dq, dk [B, T, H, 128] per value head; gates [B, T, H]
    int* d_status;
    int T, H, group, nchunks;
};

// Shared memory (bytes from a 1024-aligned base).
constexpr uint32_t R0 = 0;          // [dO ; DR] bf16 [128 x 128] (K-major A of D12);
                                    // after D12: [V' ; -R'] (A of the G_e product)
constexpr uint32_t R1 = 32768;      // B of D12, per 64-column K block (32 KB): rows 0..127
                                    // S0 (row = key channel), 128..191 V, 192..255 Uf;
                                    // after the last product, fp32 staging of du
constexpr uint32_t R2 = 98304;      // per 64-channel block (24 KB): Q, U = beta K, K rows
constexpr uint32_t R3 = 147456;     // [[P1, -P2] ; [P3, -P4]] bf16 [128 x 128]
constexpr uint32_t R4 = 180224;     // G_e, per 64-column K block (16 KB): 128 rows
constexpr uint32_t SMALL = 212992;
constexpr uint32_t SMEM_BYTES = SMALL + 8192 + 64 + 1024;
// D6 takes D12's columns 128..255 once the masked blocks have been formed;
// D7 sits in D3's columns until then
constexpr uint32_t TM_D12 = 0, TM_D6 = 128, TM_D3 = 256, TM_D7 = 256, TM_D45 = 384, TM_COLS = 512;

// fp32 row of 32 values -> 4 bf16 16-byte pieces of a K-major swizzled tile
__device__ __forceinline__ void put32(uint8_t* tile, int row, int ch0, int rows, const float* x) {
#pragma unroll
    for (int c = 0; c < 4; ++c) st_chunk(tile, sw128_chunk(row, ch0 + c, rows), x + 8 * c);
}

__global__ void __launch_bounds__(256, 1) bwd_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                              const __grid_constant__ CUtensorMap tm_k,
                                                              const __grid_constant__ CUtensorMap tm_v,
                                                              const __grid_constant__ CUtensorMap tm_do,
                                                              const __grid_constant__ CUtensorMap tm_u,
                                                              const __grid_constant__ CUtensorMap tm_dr,
                                                              const __grid_constant__ CUtensorMap tm_s0,
                                                              const __grid_constant__ CUtensorMap tm_ge,
                                                              const __grid_constant__ CUtensorMap tm_dq,
                                                              const __grid_constant__ CUtensorMap tm_dk,
                                                              const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, wg = warp >> 2, row = tid & 127;
    const int c = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int hq = h / p.group;
    const int T = p.T, H = p.H;
    const int t0 = c * C, n = min(C, T - t0);
    const size_t head = (size_t)bb * H + h;

    float* s_l = reinterpret_cast<float*>(sm + SMALL);   // [64] log2 prefix of alpha
    float* s_gam = s_l + 64;                               // [64] Gam_t
    float* s_gcr = s_l + 128;                              // [64] Gam_C / Gam_t
    float* s_beta = s_l + 192;                             // [64]
    float* s_alpha = s_l + 256;                            // [64]
    float* s_red = s_l + 320;                              // [10][64] per-token partial sums
    float* s_ge = s_l + 960;                               // [8] <G_e, S0> partials
    float* s_M = s_l + 1024;                               // [8 warps][64] column sums of M
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + SMALL + 8192);
    uint64_t* bar_mma = bar_tma + 1;
    uint64_t* bar_drain = bar_tma + 2;
    uint64_t* bar_ge = bar_tma + 3;
    uint64_t* bar_qk = bar_tma + 4;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + SMALL + 8192 + 48);
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_drain, 1);
        mbar_init(bar_ge, 1);
        mbar_init(bar_qk, 1);
        fence_barrier_init();
        // checkpoint rows: (head, chunk) -> 128 rows of a [rows, 128] view
        const int ck_row = (int)((head * p.nchunks + c) * 128);
        // the operands of D12 first, then Q and K (D7), then G_e (D6)
        mbar_expect_tx(bar_tma, 12u * 8192u);
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
            tma_load_4d(sm + R0 + blk * 16384, &tm_do, bar_tma, 64 * blk, h, t0, bb);
            tma_load_4d(sm + R0 + blk * 16384 + 8192, &tm_dr, bar_tma, 64 * blk, h, t0, bb);
            tma_load_4d(sm + R1 + blk * 32768, &tm_s0, bar_tma, 64 * blk, 0, ck_row, 0);
            tma_load_4d(sm + R1 + blk * 32768 + 8192, &tm_s0, bar_tma, 64 * blk, 0, ck_row + 64, 0);
            tma_load_4d(sm + R1 + blk * 32768 + 16384, &tm_v, bar_tma, 64 * blk, h, t0, bb);
            tma_load_4d(sm + R1 + blk * 32768 + 24576, &tm_u, bar_tma, 64 * blk, h, t0, bb);
        }
        mbar_expect_tx(bar_qk, 4u * 8192u);
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
            tma_load_4d(sm + R2 + blk * 24576, &tm_q, bar_qk, 64 * blk, hq, t0, bb);
            tma_load_4d(sm + R2 + blk * 24576 + 16384, &tm_k, bar_qk, 64 * blk, hq, t0, bb);
        }
        mbar_expect_tx(bar_ge, 4u * 8192u);
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
            tma_load_4d(sm + R4 + blk * 16384, &tm_ge, bar_ge, 64 * blk, 0, ck_row, 0);
            tma_load_4d(sm + R4 + blk * 16384 + 8192, &tm_ge, bar_ge, 64 * blk, 0, ck_row + 64, 0);
        }
    }
    if (warp == 0) tmem_alloc(s_tmem, TM_COLS);
    if (tid < C) {
        const bool valid = tid < n;
        const size_t gi = ((size_t)bb * T + t0 + min(tid, n - 1)) * H + h;
        s_alpha[tid] = valid ? __bfloat162float(p.alpha[gi]) : 1.f;
        s_beta[tid] = valid ? __bfloat162float(p.beta[gi]) : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    bool ok = true;
    uint32_t ph_mma = 0;
#define GDR_WAIT(bar, ph)                                                   \
    do {                                                                    \
        bool w_ok = mbar_wait(bar, ph);                                     \
        ph ^= 1u;                                                           \
        if (!__syncthreads_and(w_ok)) { ok = false; goto finish; }          \
    } while (0)

    // decay scan (warp 0, two tokens per lane): l, Gam, Gam_C / Gam
    if (warp == 0) {
        const int lane = tid;
        const float la0 = lg2_approx(s_alpha[2 * lane]), la1 = lg2_approx(s_alpha[2 * lane + 1]);
        float x = la0 + la1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        const float l1 = x, l0v = x - la1;
        const float last = __shfl_sync(0xffffffffu, l1, 31);  // padding adds nothing
        s_l[2 * lane] = l0v;
        s_l[2 * lane + 1] = l1;
        s_gam[2 * lane] = ex2_approx(l0v);
        s_gam[2 * lane + 1] = ex2_approx(l1);
        s_gcr[2 * lane] = ex2_approx(last - l0v);
        s_gcr[2 * lane + 1] = ex2_approx(last - l1);
    }
    {
        uint32_t ph_tma = 0;
        GDR_WAIT(bar_tma, ph_tma);
    }
    // ---- D12 = [dO ; DR] [S0 | V | Uf]^T, issued as soon as its tiles land ---------
    // (the block of the erase reads, [dO ; DR] R^T with R = Diag(beta) V - Uf, is
    // formed on the unload from the V and Uf blocks)
    if (tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, 256, 0, 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ka = (ks >> 2) * 16384u + (ks & 3) * 32u;
            const uint32_t kb = (ks >> 2) * 32768u + (ks & 3) * 32u;
            mma_bf16(tmem + TM_D12, sdesc_sw128(sbase + R0 + ka, 16, 1024),
                     sdesc_sw128(sbase + R1 + kb, 16, 1024), id, ks > 0);
        }
    }
    {
        uint32_t ph_qk = 0;
        GDR_WAIT(bar_qk, ph_qk);
    }
    // U = beta K (rows of the K tile scaled per token) next to Q and K
    {
        const int t = tid >> 2, part = tid & 3;  // token, 4 of the 16 pieces of its 128 channels
        const float f = s_beta[t];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            const int ch = part * 4 + q4, blk = ch >> 3;
            const uint32_t off = sw128_chunk(t, ch & 7, 64);
            float x[8];
            ld_chunk(sm + R2 + blk * 24576 + 16384, off, x);
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] *= f;
            st_chunk(sm + R2 + blk * 24576 + 8192, off, x);
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- D7 = [Q ; U] K^T: A rows 0..63 Q, 64..127 U (adjacent in each channel block) --
    if (tid == 0) {
        tc_fence_after();
        const uint32_t id7 = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t kq = (ks >> 2) * 24576u + (ks & 3) * 32u;
            mma_bf16(tmem + TM_D7, sdesc_sw128(sbase + R2 + kq, 16, 1024),
                     sdesc_sw128(sbase + R2 + 16384 + kq, 16, 1024), id7, ks > 0);
        }
        mma_commit(bar_mma);
    }
    GDR_WAIT(bar_mma, ph_mma);
    tc_fence_after();

    // ---- masked, decay-scaled blocks -> R3; [V' ; -R'] -> R0 ----------------------------
    {
        // lanes 0..63 (token t): dO V^T (wg 0) and dO R^T (wg 1), mask j <= t;
        // lanes 64..127: DR V^T and DR R^T, mask j < t; the R^T blocks are
        // beta_j (V^T block) - (Uf^T block)
        // M_tj of this thread's block (wg 0: u_j terms, wg 1: k_j terms), summed over
        // j < s for every s <= t, then over the warp's rows for each s
        const int t = row & 63;
        const bool strict = row >= 64;
        const float lt = s_l[t];
        const int lane = tid & 31;
        float d[32], g7[32];
        float run = 0.f;  // sum of m_j over j < 32 half
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tmem_ld32_async(tmem + lane_base + TM_D12 + 128 + wg * 64 + half * 32, d);
            tmem_ld32_async(tmem + lane_base + TM_D7 + half * 32, g7);
            if (wg) {
                float dvb[32];
                tmem_ld32_async(tmem + lane_base + TM_D12 + 128 + half * 32, dvb);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) d[e] = fmaf(s_beta[half * 32 + e], dvb[e], -d[e]);
            } else {
                tmem_wait_ld();
            }
            float x[32], m[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int j = half * 32 + e;
                const bool keep = strict ? j < t : j <= t;
                const float v = keep ? d[e] * ex2_approx(fminf(lt - s_l[j], 0.f)) : 0.f;
                x[e] = wg ? -v : v;
                m[e] = wg ? -g7[e] * v : s_beta[j] * g7[e] * v;
            }
            put32(sm + R3, row, wg * 8 + half * 4, 128, x);
            // R(s) = sum_{j < s} m_j for s = half * 32 + e (zero for s > t)
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float r_s = run;
                run += m[e];
                m[e] = half * 32 + e <= t ? r_s : 0.f;
            }
            const float cs = warp_colsum32(m, lane);
            s_M[warp * 64 + half * 32 + lane] = cs;
        }
    }
    {
        // rows t of V and R = beta V - Uf scaled by Gam_C / Gam_t (R negated) -> R0
        const int t = tid >> 2, part = tid & 3;
        const float f = s_gcr[t], fb = f * s_beta[t];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            const int ch = part * 4 + q4;
            float y[8], u[8];
            ld_chunk(sm + R1, sw128_chunk(128 + t, ch, 256), y);
            ld_chunk(sm + R1, sw128_chunk(192 + t, ch, 256), u);
#pragma unroll
            for (int e = 0; e < 8; ++e) u[e] = fmaf(f, u[e], -fb * y[e]);
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] *= f;
            st_chunk(sm + R0, sw128_chunk(t, ch, 128), y);
            st_chunk(sm + R0, sw128_chunk(64 + t, ch, 128), u);
        }
    }
    fence_proxy_async();
    tc_fence_before();
    {
        uint32_t ph_ge = 0;  // G_e (loaded at the start) has landed
        GDR_WAIT(bar_ge, ph_ge);
    }

    // ---- D3 = P [U ; K];  D45 = P^T [Q ; U];  D6 = [V' ; -R'] G_e^T ----------------
    if (tid == 0) {
        tc_fence_after();
        const uint32_t id3 = idesc_bf16(128, 128, 0, 1);
        const uint32_t id4 = idesc_bf16(128, 128, 1, 1);
        const uint32_t id5 = idesc_bf16(128, 128, 0, 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_D3, sdesc_sw128(sbase + R3 + (ks >> 2) * 16384u + (ks & 3) * 32u, 16, 1024),
                     sdesc_sw128(sbase + R2 + 8192 + ks * 2048u, 24576, 1024), id3, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_D45, sdesc_sw128(sbase + R3 + ks * 2048u, 16384, 1024),
                     sdesc_sw128(sbase + R2 + ks * 2048u, 24576, 1024), id4, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + TM_D6, sdesc_sw128(sbase + R0 + (ks >> 2) * 16384u + (ks & 3) * 32u, 16, 1024),
                     sdesc_sw128(sbase + R4 + (ks >> 2) * 16384u + (ks & 3) * 32u, 16, 1024), id5, ks > 0);
        mma_commit(bar_mma);
    }
    // <G_e, S0> over the whole state, from the two tiles in shared memory (the
    // same 128-byte swizzle at 1024-aligned bases pairs equal elements)
    {
        float acc = 0.f;
#pragma unroll 4
        for (int i = tid; i < 2048; i += 256) {
            const uint32_t blk = (uint32_t)i >> 10, o = ((uint32_t)i & 1023u) * 16u;
            float a[8], b[8];
            ld_chunk(sm + R4 + blk * 16384, o, a);
            ld_chunk(sm + R1 + blk * 32768, o, b);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc = fmaf(a[e], b[e], acc);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if ((tid & 31) == 0) s_ge[warp] = acc;
    }
    GDR_WAIT(bar_mma, ph_mma);
    tc_fence_after();

    // ---- epilogue -------------------------------------------------------------------
    // Warps w and w + 2 of a warpgroup cover the same tokens and columns: the
    // first (TMEM lanes 0..63: dq rows) stages du = D45 + D6 for the second
    // (lanes 64..127: dk rows) and signals a barrier of the pair; then both
    // form their gradients at the same time. dq and dk leave as fp32 tiles by
    // TMA (32 columns x 64 tokens, 128-byte swizzle) from R3 and R0, whose
    // operands the finished products no longer need; rows past T are not
    // written.
    {
        auto stage = [&](uint8_t* box, int t_, const float* x) {
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<float4*>(box + t_ * 128 + ((c ^ (t_ & 7)) << 4)) =
                    make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
        };
        float* du_f = reinterpret_cast<float*>(sm + R1);  // [64][128 + 4] fp32 (R1 is free)
        constexpr int DUP = 132;
        const int t = row & 63;
        const float gam = s_gam[t], be = s_beta[t];
        const uint32_t pair_bar = 1u + (uint32_t)(wg * 2 + (warp & 1));
        if (row < 64) {
            // du -> du_f and the sum u du^G
            float red_g = 0.f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int i0 = wg * 64 + half * 32;
                float du[32], dg[32], kv[32];
                tmem_ld32_async(tmem + lane_base + TM_D45 + i0, du);
                tmem_ld32_async(tmem + lane_base + TM_D6 + i0, dg);
                tmem_wait_ld();
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int ch = (i0 >> 3) + c4, blk = ch >> 3;
                    ld_chunk(sm + R2 + blk * 24576 + 16384, sw128_chunk(t, ch & 7, 64), kv + 8 * c4);
                }
#pragma unroll
                for (int e = 0; e < 32; ++e) red_g = fmaf(be * kv[e], dg[e], red_g);
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4*>(du_f + t * DUP + i0 + e) =
                        make_float4(du[e] + dg[e], du[e + 1] + dg[e + 1], du[e + 2] + dg[e + 2], du[e + 3] + dg[e + 3]);
            }
            __threadfence_block();
            named_bar_arrive(pair_bar, 64);
            s_red[(6 + wg) * 64 + t] = red_g;
            // dq = Gam dO S0^T + D3 and the sum q . (dO S0^T)
            float red_a = 0.f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int i0 = wg * 64 + half * 32;
                float x1[32], d3[32], qv[32];
                tmem_ld32_async(tmem + lane_base + TM_D12 + i0, x1);
                tmem_ld32_async(tmem + lane_base + TM_D3 + i0, d3);
                tmem_wait_ld();
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int ch = (i0 >> 3) + c4, blk = ch >> 3;
                    ld_chunk(sm + R2 + blk * 24576, sw128_chunk(t, ch & 7, 64), qv + 8 * c4);
                }
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    red_a = fmaf(qv[e], x1[e], red_a);
                    x1[e] = fmaf(gam, x1[e], d3[e]);
                }
                stage(sm + R3 + (i0 >> 5) * 8192, t, x1);
            }
            s_red[(0 + wg) * 64 + t] = gam * red_a;
        } else {
            // de = Gam DR S0^T + D3; dkr = D45 + D6; dk = dkr + beta (de + du);
            // sums e . (dr S0^T), k dkr^G and k (de + du)
            named_bar_sync(pair_bar, 64);
            float red_db = 0.f, red_l = 0.f, red_g = 0.f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int i0 = wg * 64 + half * 32;
                float x2[32], d3[32], dkr[32], dg[32];
                tmem_ld32_async(tmem + lane_base + TM_D12 + i0, x2);
                tmem_ld32_async(tmem + lane_base + TM_D3 + i0, d3);
                tmem_ld32_async(tmem + lane_base + TM_D45 + i0, dkr);
                tmem_ld32_async(tmem + lane_base + TM_D6 + i0, dg);
                tmem_wait_ld();
                float kv[32];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int ch = (i0 >> 3) + c4, blk = ch >> 3;
                    ld_chunk(sm + R2 + blk * 24576 + 16384, sw128_chunk(t, ch & 7, 64), kv + 8 * c4);
                }
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 du4 = *reinterpret_cast<const float4*>(du_f + t * DUP + i0 + e);
                    const float du[4] = {du4.x, du4.y, du4.z, du4.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float de = fmaf(gam, x2[e + q], d3[e + q]);
                        red_db = fmaf(kv[e + q], de + du[q], red_db);
                        red_l = fmaf(kv[e + q], x2[e + q], red_l);  // k . (dr S0^T)
                        red_g = fmaf(kv[e + q], dg[e + q], red_g);
                        x2[e + q] = fmaf(be, de + du[q], dkr[e + q] + dg[e + q]);
                    }
                }
                stage(sm + R0 + (i0 >> 5) * 8192, t, x2);
            }
            s_red[(2 + wg) * 64 + t] = gam * be * red_l;
            s_red[(4 + wg) * 64 + t] = red_db;
            s_red[(8 + wg) * 64 + t] = red_g;
        }
        fence_proxy_async();
        __syncthreads();
        if (tid == 32) {
#pragma unroll
            for (int box = 0; box < 4; ++box) {
                tma_store_4d(&tm_dq, sm + R3 + box * 8192, 32 * box, h, t0, bb);
                tma_store_4d(&tm_dk, sm + R0 + box * 8192, 32 * box, h, t0, bb);
            }
            bulk_commit_group();
        }
        if (warp == 0) {
            // dlam_s = sum_{t >= s} a_t + sum_{t >= s, j < s} M_tj + Gam_C <G_e, S0>
            //         + sum_{j < s} c_j: lane l holds s = 2l, 2l + 1; a suffix
            // scan of a and an exclusive prefix scan of c over the lanes
            const int lane = tid, s0 = 2 * lane, s1 = s0 + 1;
            auto a_of = [&](int u) {
                return u < n ? s_red[u] + s_red[64 + u] + s_red[128 + u] + s_red[192 + u] : 0.f;
            };
            auto c_of = [&](int j) { return s_red[384 + j] + s_red[448 + j] + s_red[512 + j] + s_red[576 + j]; };
            const float a0 = a_of(s0), a1 = a_of(s1), c0 = c_of(s0), c1 = c_of(s1);
            float suf = a0 + a1, pre = c0 + c1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float ys = __shfl_down_sync(0xffffffffu, suf, off);
                const float yp = __shfl_up_sync(0xffffffffu, pre, off);
                if (lane + off < 32) suf += ys;
                if (lane >= off) pre += yp;
            }
            pre -= c0 + c1;  // exclusive: sum over j < s0
            float ge = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) ge += s_ge[w];
            const float base = s_gam[C - 1] * ge;  // padding tokens decay by 1: Gam_{63} = Gam_{n-1}
            float m0 = 0.f, m1 = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                m0 += s_M[w * 64 + s0];
                m1 += s_M[w * 64 + s1];
            }
            const float cum0 = base + m0 + suf + pre;
            const float cum1 = base + m1 + (suf - a0) + (pre + c0);
            const size_t gi = ((size_t)bb * T + t0 + s0) * H + h;
            if (s0 < n) {
                p.dalpha[gi] = cum0 / s_alpha[s0];
                p.db[gi] = s_red[256 + s0] + s_red[320 + s0];
            }
            if (s1 < n) {
                p.dalpha[gi + H] = cum1 / s_alpha[s1];
                p.db[gi + H] = s_red[256 + s1] + s_red[320 + s1];
            }
        }
    }

    if (tid == 32) bulk_wait_group_read0();
finish:
    if (!ok && tid == 0) {
        // before the block leaves (each wait bounded): the input copies have
        // landed and every issued MMA has finished
        (void)mbar_wait(bar_tma, 0);
        (void)mbar_wait(bar_qk, 0);
        (void)mbar_wait(bar_ge, 0);
        mma_commit(bar_drain);
        (void)mbar_wait(bar_drain, 0);
        flag_status(p.d_status, GDR_DEVICE_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
#undef GDR_WAIT
}

}  // namespace bwdtc

// maps: q, k (q/k heads), v, dO (value heads), bf16 [B, T, H, 128] each.
// ck_maps: U = beta v - r and dr (bf16 [B, T, H, 128]), the chunk-start states
// and the chunk-end state gradients (bf16 [B, H, nchunks, 128, 128], each
// mapped as one [B H nchunks 128, 128] view), then dq and dk (fp32
// [B, T, H, 128], box 32 x 64 tokens, for the tile stores).
cudaError_t launch_bwd_chunk_tc(const CUtensorMap* maps, const CUtensorMap* ck_maps, const void* alpha,
                                const void* beta, float* dq, float* dk, float* dalpha, float* db,
                                int* d_status, int B, int T, int H, int group, int nchunks,
                                cudaStream_t st) {
    using namespace bwdtc;
    TcParams p;
    p.alpha = reinterpret_cast<const __nv_bfloat16*>(alpha);
    p.beta = reinterpret_cast<const __nv_bfloat16*>(beta);
    p.dq = dq; p.dk = dk; p.dalpha = dalpha; p.db = db; p.d_status = d_status;
    p.T = T; p.H = H; p.group = group; p.nchunks = nchunks;
    cudaError_t e = cudaFuncSetAttribute(bwd_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    bwd_chunk_tc_kernel<<<dim3(nchunks, H, B), 256, SMEM_BYTES, st>>>(maps[0], maps[1], maps[2], maps[3], ck_maps[0],
                                                                    ck_maps[1], ck_maps[2], ck_maps[3], ck_maps[4],
                                                                    ck_maps[5], p);
    return cudaGetLastError();
}

}  // namespace gdr
