// One decode step of the gated delta rule per head, streaming the fp32 state
// through HBM once (read, update in registers, write back in place).
//
// With S' = Diag(alpha) S, r = (b.k) S' and S_new = S' - k^T r + (w.k)^T v
// ("Recurrent Memory: Write, Erase, Decay, Read", sections 03-05; gates per
// "Erase-then-Delta Attention", abstract), the read o = q S_new expands to
//   o = (q.alpha) S - (q.k) r + (q.(w.k)) v,   r = (b.k.alpha) S,
// so one pass over S gives both column reductions, and S_new is written from
// the registers that hold S.
#include "common.cuh"

namespace gdr {

// Block: 256 threads per head. Threads are laid out as RPP row lanes x TPR
// column groups of 4 floats (one 16-byte load each); a warp reads contiguous
// 16-byte pieces of one or more rows. Each thread keeps NR rows x 4 columns.
// A block handles DV value columns of one head (blockIdx.y selects which DV of
// the head's dvf): every column's reductions over d_k stay inside its block,
// so a wide head can be split over blocks with no exchange between them.
// Two resident blocks per SM (128 registers a thread) up to 16 state rows per
// thread; 32 rows (128 registers of state alone) take one.
template <typename TI, int DV, int NR>
__global__ void __launch_bounds__(256, NR <= 16 ? 2 : 1) decode_step_kernel(
    const TI* __restrict__ q, const TI* __restrict__ k, const TI* __restrict__ v,
    const TI* __restrict__ alpha, const TI* __restrict__ bg, const TI* __restrict__ wg, int akind,
    int bkind, int wkind, float* __restrict__ S, TI* __restrict__ o, int dk, int dvf, int group) {
    constexpr int TPR = DV / 4;
    constexpr int RPP = 256 / TPR;
    const int bh = blockIdx.x;
    const int c0 = blockIdx.y * DV;  // this block's first value column
    const int tid = threadIdx.x;
    __shared__ float s_alpha[256], s_eka[256], s_qa[256], s_k[256], s_wk[256];
    __shared__ float s_v[DV];
    __shared__ float4 s_red[2][RPP][TPR];
    __shared__ float s_dots[2];

    // Launched as a programmatic dependent of the previous work on the stream:
    // the next step's blocks may be scheduled once every block of this one has
    // started, and nothing is read before the previous grid has completed and
    // its writes (the state of the previous step, this step's inputs) are visible.
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const size_t bhq = (size_t)(bh / group);  // q, k have H / group heads
    for (int i = tid; i < dk; i += 256) {
        const size_t gi = (size_t)bh * dk + i;
        float ki = to_f32(k[bhq * dk + i]), qi = to_f32(q[bhq * dk + i]);
        float a = akind == GDR_GATE_NONE ? 1.f
                  : akind == GDR_GATE_SCALAR ? to_f32(alpha[bh]) : to_f32(alpha[gi]);
        float bb = bkind == GDR_GATE_NONE ? 0.f
                   : bkind == GDR_GATE_SCALAR ? to_f32(bg[bh]) : to_f32(bg[gi]);
        float ww = wkind == GDR_GATE_TIED ? bb
                   : wkind == GDR_GATE_NONE ? 1.f
                   : wkind == GDR_GATE_SCALAR ? to_f32(wg[bh]) : to_f32(wg[gi]);
        s_alpha[i] = a;
        s_eka[i] = bb * ki * a;
        s_qa[i] = qi * a;
        s_k[i] = ki;
        s_wk[i] = ww * ki;
    }
    for (int j = tid; j < DV; j += 256) s_v[j] = to_f32(v[(size_t)bh * dvf + c0 + j]);
    __syncthreads();
    if (tid < 32) {
        float d1 = 0.f, d2 = 0.f;
        for (int i = tid; i < dk; i += 32) {
            float qi = to_f32(q[bhq * dk + i]);
            d1 += qi * s_k[i];
            d2 += qi * s_wk[i];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            d1 += __shfl_xor_sync(0xffffffffu, d1, off);
            d2 += __shfl_xor_sync(0xffffffffu, d2, off);
        }
        if (tid == 0) {
            s_dots[0] = d1;
            s_dots[1] = d2;
        }
    }

    const int cg = tid % TPR, rl = tid / TPR;
    float4* Sh = reinterpret_cast<float4*>(S + (size_t)bh * dk * dvf + c0);
    const size_t rstride = (size_t)dvf / 4;  // float4 per state row
    float4 sv[NR];
    float4 racc = make_float4(0.f, 0.f, 0.f, 0.f), aacc = racc;
#pragma unroll
    for (int m = 0; m < NR; ++m) {
        const int row = rl + RPP * m;
        if (row < dk) sv[m] = __ldcs(Sh + (size_t)row * rstride + cg);
        else sv[m] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int m = 0; m < NR; ++m) {
        const int row = rl + RPP * m;
        if (row < dk) {
            const float e = s_eka[row], qa = s_qa[row];
            racc.x += e * sv[m].x; racc.y += e * sv[m].y; racc.z += e * sv[m].z; racc.w += e * sv[m].w;
            aacc.x += qa * sv[m].x; aacc.y += qa * sv[m].y; aacc.z += qa * sv[m].z; aacc.w += qa * sv[m].w;
        }
    }
    s_red[0][rl][cg] = racc;
    s_red[1][rl][cg] = aacc;
    __syncthreads();
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int l = 0; l < RPP; ++l) {
        float4 p = s_red[0][l][cg];
        r.x += p.x; r.y += p.y; r.z += p.z; r.w += p.w;
    }
    const float4 v4 = make_float4(s_v[4 * cg], s_v[4 * cg + 1], s_v[4 * cg + 2], s_v[4 * cg + 3]);
#pragma unroll
    for (int m = 0; m < NR; ++m) {
        const int row = rl + RPP * m;
        if (row < dk) {
            const float a = s_alpha[row], kk = s_k[row], wk = s_wk[row];
            float4 n;
            n.x = a * sv[m].x - kk * r.x + wk * v4.x;
            n.y = a * sv[m].y - kk * r.y + wk * v4.y;
            n.z = a * sv[m].z - kk * r.z + wk * v4.z;
            n.w = a * sv[m].w - kk * r.w + wk * v4.w;
            __stcs(Sh + (size_t)row * rstride + cg, n);
        }
    }
    if (rl == 0) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int l = 0; l < RPP; ++l) {
            float4 p = s_red[1][l][cg];
            a.x += p.x; a.y += p.y; a.z += p.z; a.w += p.w;
        }
        const float qk = s_dots[0], qwk = s_dots[1];
        TI* ob = o + (size_t)bh * dvf + c0 + 4 * cg;
        ob[0] = from_f32<TI>(a.x - qk * r.x + qwk * v4.x);
        ob[1] = from_f32<TI>(a.y - qk * r.y + qwk * v4.y);
        ob[2] = from_f32<TI>(a.z - qk * r.z + qwk * v4.z);
        ob[3] = from_f32<TI>(a.w - qk * r.w + qwk * v4.w);
    }
}

template <typename TI, int DV>
static cudaError_t launch_decode_dv(const void* q, const void* k, const void* v, const void* a,
                                    const void* b, const void* w, int ak, int bk, int wk, float* S,
                                    void* o, int BH, int dk, int dvf, int group, cudaStream_t st) {
    constexpr int RPP = 256 / (DV / 4);
    const int nr = (dk + RPP - 1) / RPP;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(BH, dvf / DV);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap the previous tail
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
#define GDR_DEC(NRV)                                                                                  \
    e = cudaLaunchKernelEx(&cfg, decode_step_kernel<TI, DV, NRV>, (const TI*)q, (const TI*)k,        \
                           (const TI*)v, (const TI*)a, (const TI*)b, (const TI*)w, ak, bk, wk, S,     \
                           (TI*)o, dk, dvf, group)
    if (nr <= 4) GDR_DEC(4);
    else if (nr <= 8) GDR_DEC(8);
    else if (nr <= 16) GDR_DEC(16);
    else if (nr <= 32) GDR_DEC(32);
    else return cudaErrorInvalidValue;
#undef GDR_DEC
    return e;
}

// Rows per thread needed for (d_k, d_v); the launcher supports up to 32.
// Value columns per block: the whole head, except d_v = 256 with d_k > 128
// (64 state rows per thread), which takes two blocks of 128 columns.
int decode_cols_per_block(int dk, int dv) { return dv == 256 && dk > 128 ? 128 : dv; }

int decode_rows_per_thread(int dk, int dv) {
    int rpp = 256 / (decode_cols_per_block(dk, dv) / 4);
    return (dk + rpp - 1) / rpp;
}

template <typename TI>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const void* a,
                                   const void* b, const void* w, int ak, int bk, int wk, float* S,
                                   void* o, int BH, int dk, int dv, int group, cudaStream_t st) {
    switch (dv) {
        case 16: return launch_decode_dv<TI, 16>(q, k, v, a, b, w, ak, bk, wk, S, o, BH, dk, dv, group, st);
        case 32: return launch_decode_dv<TI, 32>(q, k, v, a, b, w, ak, bk, wk, S, o, BH, dk, dv, group, st);
        case 64: return launch_decode_dv<TI, 64>(q, k, v, a, b, w, ak, bk, wk, S, o, BH, dk, dv, group, st);
        case 128: return launch_decode_dv<TI, 128>(q, k, v, a, b, w, ak, bk, wk, S, o, BH, dk, dv, group, st);
        case 256:
            return decode_cols_per_block(dk, dv) == 256
                       ? launch_decode_dv<TI, 256>(q, k, v, a, b, w, ak, bk, wk, S, o, BH, dk, dv, group, st)
                       : launch_decode_dv<TI, 128>(q, k, v, a, b, w, ak, bk, wk, S, o, BH, dk, dv, group, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* a, const void* b,
                          const void* w, int ak, int bk, int wk, float* S, void* o, int BH, int dk,
                          int dv, int dtype, int group, cudaStream_t st) {
    if (dtype == GDR_BF16)
        return launch_decode_t<__nv_bfloat16>(q, k, v, a, b, w, ak, bk, wk, S, o, BH, dk, dv, group, st);
    return launch_decode_t<float>(q, k, v, a, b, w, ak, bk, wk, S, o, BH, dk, dv, group, st);
}

}  // namespace gdr
