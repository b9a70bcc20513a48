// Exact fp32 forward pass, one token at a time, on CUDA cores.
//
// Used for fp32 inputs (where bf16/tf32 tensor-core operands cannot hold a
// 1e-4 relative error) and for shapes outside the tensor-core chunk kernel.
// Per token: S <- Diag(alpha) S; r = (b.k) S; S <- S - k^T r + (w.k)^T v;
// o = q S ("Recurrent Memory: Write, Erase, Decay, Read", sections 01-05;
// "Erase-then-Delta Attention", abstract).
//
// Columns of S evolve independently (the erase acts from the left), so a
// thread owns one column j of one head's state, d_k values in registers.
#include "common.cuh"

namespace gdr {

constexpr int kRecCols = 64;  // threads (state columns) per block

// MAXDK: the state column a thread holds in registers (128, or 256 for the
// wider heads, where part of it lives in local memory).
template <typename TI, int kRecMaxDK>
__global__ void __launch_bounds__(kRecCols) recurrent_fwd_kernel(
    const TI* __restrict__ q, const TI* __restrict__ k, const TI* __restrict__ v,
    const TI* __restrict__ alpha, const TI* __restrict__ bg, const TI* __restrict__ wg, int akind,
    int bkind, int wkind, const float* __restrict__ S0, TI* __restrict__ o, float* __restrict__ ST,
    int T, int H, int dk, int dv, int group) {
    const int b = blockIdx.z, h = blockIdx.y;
    const int j = blockIdx.x * kRecCols + threadIdx.x;
    const bool col_ok = j < dv;
    __shared__ float s_a[2][kRecMaxDK], s_bk[2][kRecMaxDK], s_k[2][kRecMaxDK], s_wk[2][kRecMaxDK],
        s_q[2][kRecMaxDK];

    float s[kRecMaxDK];
    const size_t head = (size_t)b * H + h;
#pragma unroll
    for (int i = 0; i < kRecMaxDK; ++i)
        s[i] = (S0 && col_ok && i < dk) ? S0[(head * dk + i) * dv + j] : 0.f;

    for (int t = 0; t < T; ++t) {
        const int buf = t & 1;
        const size_t tok = ((size_t)b * T + t) * H + h;
        const size_t tokq = ((size_t)b * T + t) * (H / group) + h / group;  // q, k have H / group heads
        for (int i = threadIdx.x; i < dk; i += kRecCols) {
            const size_t gi = tok * dk + i;
            const size_t qi = tokq * dk + i;
            float ki = to_f32(k[qi]);
            float a = akind == GDR_GATE_NONE ? 1.f
                      : akind == GDR_GATE_SCALAR ? to_f32(alpha[tok]) : to_f32(alpha[gi]);
            float bb = bkind == GDR_GATE_NONE ? 0.f
                       : bkind == GDR_GATE_SCALAR ? to_f32(bg[tok]) : to_f32(bg[gi]);
            float ww = wkind == GDR_GATE_TIED ? bb
                       : wkind == GDR_GATE_NONE ? 1.f
                       : wkind == GDR_GATE_SCALAR ? to_f32(wg[tok]) : to_f32(wg[gi]);
            s_a[buf][i] = a;
            s_bk[buf][i] = bb * ki;
            s_k[buf][i] = ki;
            s_wk[buf][i] = ww * ki;
            s_q[buf][i] = to_f32(q[qi]);
        }
        __syncthreads();  // double buffering makes one barrier per token enough
        const float vj = col_ok ? to_f32(v[tok * dv + j]) : 0.f;
        float r = 0.f;
#pragma unroll
        for (int i = 0; i < kRecMaxDK; ++i) {
            if (i < dk) {
                s[i] *= s_a[buf][i];
                r += s_bk[buf][i] * s[i];
            }
        }
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < kRecMaxDK; ++i) {
            if (i < dk) {
                s[i] += -s_k[buf][i] * r + s_wk[buf][i] * vj;
                acc += s_q[buf][i] * s[i];
            }
        }
        if (col_ok) o[tok * dv + j] = from_f32<TI>(acc);
    }
    if (ST && col_ok) {
#pragma unroll
        for (int i = 0; i < kRecMaxDK; ++i)
            if (i < dk) ST[(head * dk + i) * dv + j] = s[i];
    }
}

cudaError_t launch_recurrent(const void* q, const void* k, const void* v, const void* a,
                             const void* b, const void* w, int ak, int bk, int wk, const float* S0,
                             void* o, float* ST, int B, int T, int H, int dk, int dv, int dtype,
                             int group, cudaStream_t st) {
    dim3 grid((dv + kRecCols - 1) / kRecCols, H, B);
    auto go = [&](auto kern, auto tag) {
        using TI = decltype(tag);
        kern<<<grid, kRecCols, 0, st>>>((const TI*)q, (const TI*)k, (const TI*)v, (const TI*)a,
                                        (const TI*)b, (const TI*)w, ak, bk, wk, S0, (TI*)o, ST, T, H,
                                        dk, dv, group);
    };
    if (dtype == GDR_BF16) {
        if (dk <= 128) go(recurrent_fwd_kernel<__nv_bfloat16, 128>, __nv_bfloat16{});
        else go(recurrent_fwd_kernel<__nv_bfloat16, 256>, __nv_bfloat16{});
    } else {
        if (dk <= 128) go(recurrent_fwd_kernel<float, 128>, float{});
        else go(recurrent_fwd_kernel<float, 256>, float{});
    }
    return cudaGetLastError();
}

}  // namespace gdr
