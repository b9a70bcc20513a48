// C ABI entry points (include/gdr.h): argument checks on the host, TMA tensor
// maps for the tensor-core path, and dispatch to the kernels.
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "common.cuh"

namespace gdr {
cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* a, const void* b,
                          const void* w, int ak, int bk, int wk, float* S, void* o, int BH, int dk,
                          int dv, int dtype, int group, cudaStream_t st);
int decode_rows_per_thread(int dk, int dv);
cudaError_t launch_recurrent(const void* q, const void* k, const void* v, const void* a,
                             const void* b, const void* w, int ak, int bk, int wk, const float* S0,
                             void* o, float* ST, int B, int T, int H, int dk, int dv, int dtype,
                             int group, cudaStream_t st);
cudaError_t launch_chunk_erasefree_sm100(const CUtensorMap* maps, const void* q, const void* k,
                                         const void* v, const void* alpha, const void* w,
                                         int akind, int wkind, const float* S0, void* o, float* ST,
                                         int* d_status, int B, int T, int H, int dv, int group,
                                         cudaStream_t st);
size_t twopass_workspace_bytes(int B, int T, int H, int dv);
cudaError_t launch_chunk_twopass_gdn(const CUtensorMap* maps, const CUtensorMap* ws_maps, void* ws,
                                     const void* alpha, const void* beta, const float* S0, void* o,
                                     float* ST, int* d_status, int B, int T, int H, int dv, int group,
                                     cudaStream_t st, __nv_bfloat16* ckS = nullptr, __nv_bfloat16* up = nullptr);
size_t twopass256_workspace_bytes(int B, int T, int H, int dv);
cudaError_t launch_chunk_twopass_gdn256(const CUtensorMap* maps, const CUtensorMap* ws_maps,
                                        const void* alpha, const void* beta, const float* S0, void* o,
                                        float* ST, int* d_status, int B, int T, int H, int dv, int group,
                                        cudaStream_t st);
size_t twopass_general_workspace_bytes(int B, int T, int H, int dv, bool untied);
cudaError_t launch_chunk_twopass_general(const CUtensorMap* maps,
                                         bool (*make_map)(CUtensorMap*, const void*, int, int, int, int),
                                         void* ws, const void* q, const void* k, const void* v,
                                         const void* alpha,
                                         const void* b, const void* w, int akind, int bkind,
                                         int wkind, const float* S0, void* o, float* ST,
                                         int* d_status, int B, int T, int H, int dv, int group,
                                         bool allow_segments, cudaStream_t st);
cudaError_t launch_chunk_sm100(const CUtensorMap* maps, const void* q, const void* k, const void* v,
                               const void* alpha, const void* b,
                               const void* w, int akind, int bkind, int wkind, bool tied,
                               const float* S0, void* o, float* ST, int* d_status, int B, int T,
                               int H, int dv, int group, cudaStream_t st);
}  // namespace gdr

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool kind_ok(int kind, bool allow_tied) {
    return kind == GDR_GATE_NONE || kind == GDR_GATE_SCALAR || kind == GDR_GATE_CHANNEL ||
           (allow_tied && kind == GDR_GATE_TIED);
}

// Pointer must be NULL exactly when the gate carries no data of its own.
bool gate_ptr_ok(int kind, const void* p) {
    bool needs = kind == GDR_GATE_SCALAR || kind == GDR_GATE_CHANNEL;
    return needs ? p != nullptr : p == nullptr;
}

// 4-D map over a [B, T, H, d] bf16 tensor, box {64 (d), 1 (H), 64 (T), 1 (B)},
// 128-byte swizzle, zero fill outside the tensor (masks the last chunk).
bool make_map(CUtensorMap* m, const void* base, int B, int T, int H, int d) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

namespace gdr {
bool make_tma_map_bf16(CUtensorMap* m, const void* base, int B, int T, int H, int d) {
    return make_map(m, base, B, T, H, d);
}

// 4-D map over a [B, T, H, d] fp32 tensor, box {32 (d), 1 (H), 64 (T), 1 (B)}
// (128-byte rows), 128-byte swizzle: the tile stores of fp32 outputs.
bool make_tma_map_f32(CUtensorMap* m, const void* base, int B, int T, int H, int d) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 4, (cuuint64_t)H * d * 4, (cuuint64_t)T * H * d * 4};
    cuuint32_t box[4] = {32, 1, 64, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}
}  // namespace gdr

namespace {

// Two-pass paths (per-chunk factors of all chunks in parallel, then the state
// pass) exist for the tensor-core shape with an erase gate and d_v <= 128:
// the Gated DeltaNet form (scalar decay, tied scalar beta) has its own pair of
// kernels, every other gate form the general pair. At d_k = 256 the Gated
// DeltaNet form has a pair of its own (d_v a multiple of 64 up to 256).
enum TwoPass { TP_NONE = 0, TP_GDN = 1, TP_GENERAL = 2, TP_GDN256 = 3 };

TwoPass twopass_kind(int T, int d_k, int d_v, int ak, int bk, int wk, int dtype) {
    if (T <= 0 || dtype != GDR_BF16) return TP_NONE;
    const bool gdn = ak == GDR_GATE_SCALAR && bk == GDR_GATE_SCALAR && wk == GDR_GATE_TIED;
    if (d_k == 256) return gdn && d_v % 64 == 0 && d_v >= 64 && d_v <= 256 ? TP_GDN256 : TP_NONE;
    if (d_k != 128 || !(d_v == 64 || d_v == 128)) return TP_NONE;
    if (bk == GDR_GATE_NONE) return TP_NONE;  // erase-free: single pass, no solve
    if (gdn) return TP_GDN;
    return TP_GENERAL;
}

size_t twopass_bytes(TwoPass kind, int B, int T, int H, int d_v, int bk, int wk) {
    if (kind == TP_GDN) return gdr::twopass_workspace_bytes(B, T, H, d_v);
    if (kind == TP_GDN256) return gdr::twopass256_workspace_bytes(B, T, H, d_v);
    if (kind == TP_GENERAL)
        return gdr::twopass_general_workspace_bytes(B, T, H, d_v,
                                                    !(wk == GDR_GATE_TIED && bk == GDR_GATE_SCALAR));
    return 0;
}

}  // namespace

extern "C" {

size_t gdr_chunk_fwd_workspace_size(int B, int T, int H, int d_k, int d_v, int alpha_kind,
                                    int b_kind, int w_kind, int dtype) {
    if (B < 1 || H < 1) return 0;
    return twopass_bytes(twopass_kind(T, d_k, d_v, alpha_kind, b_kind, w_kind, dtype), B, T, H, d_v,
                         b_kind, w_kind);
}

const char* gdr_status_string(int s) {
    switch (s) {
        case GDR_OK: return "GDR_OK";
        case GDR_ERR_INVALID_ARG: return "GDR_ERR_INVALID_ARG";
        case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED";
        case GDR_ERR_MISALIGNED: return "GDR_ERR_MISALIGNED";
        case GDR_ERR_LAUNCH: return "GDR_ERR_LAUNCH";
        case GDR_ERR_NO_DEVICE: return "GDR_ERR_NO_DEVICE";
        default: return "GDR_ERR_UNKNOWN";
    }
}

int gdr_version(void) { return (1 << 16) | 0; }

}  // extern "C"

namespace gdr {

// gdr_chunk_fwd_grouped with one more switch: allow_segments = false keeps the
// general two-pass path on the caller's stream alone (no auxiliary stream or
// events are created or used).
gdr_status chunk_fwd_impl(const void* q, const void* k, const void* v, const void* alpha,
                          const void* b, const void* w, int alpha_kind, int b_kind, int w_kind,
                          const float* S0, void* o, float* S_T, void* workspace,
                          size_t workspace_bytes, int B, int T, int H_qk, int H, int d_k, int d_v,
                          int chunk, int dtype, int* d_status, bool allow_segments, void* stream) {
    if (B < 1 || H < 1 || T < 0 || d_k < 1 || d_v < 1) return GDR_ERR_INVALID_ARG;
    if (H_qk < 1 || H % H_qk != 0) return GDR_ERR_INVALID_ARG;
    const int group = H / H_qk;
    if (dtype != GDR_BF16 && dtype != GDR_FP32) return GDR_ERR_INVALID_ARG;
    if (!kind_ok(alpha_kind, false) || !kind_ok(b_kind, false) || !kind_ok(w_kind, true))
        return GDR_ERR_INVALID_ARG;
    // with T = 0 there are no token arrays (zero-length buffers may be NULL)
    if (T > 0 && (!gate_ptr_ok(alpha_kind, alpha) || !gate_ptr_ok(b_kind, b) ||
                  !gate_ptr_ok(w_kind, w)))
        return GDR_ERR_INVALID_ARG;
    if (w_kind == GDR_GATE_TIED && b_kind == GDR_GATE_NONE) return GDR_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !o)) return GDR_ERR_INVALID_ARG;
    if (chunk != 64) return GDR_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t state_bytes = (size_t)B * H * d_k * d_v * sizeof(float);
    if (T == 0) {
        if (!S_T) return GDR_OK;
        cudaError_t e = S0 ? (S0 == S_T ? cudaSuccess
                                        : cudaMemcpyAsync(S_T, S0, state_bytes,
                                                          cudaMemcpyDeviceToDevice, st))
                           : cudaMemsetAsync(S_T, 0, state_bytes, st);
        return e == cudaSuccess ? GDR_OK : GDR_ERR_LAUNCH;
    }
    const bool tc_path = dtype == GDR_BF16 && d_k == 128 && d_v % 64 == 0;
    if (!tc_path && (d_k > 256 || d_v > 1024)) return GDR_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
        (S0 && !aligned16(S0)) || (S_T && !aligned16(S_T)))
        return GDR_ERR_MISALIGNED;
    if ((alpha_kind == GDR_GATE_CHANNEL && !aligned16(alpha)) ||
        (b_kind == GDR_GATE_CHANNEL && !aligned16(b)) ||
        (w_kind == GDR_GATE_CHANNEL && !aligned16(w)))
        return GDR_ERR_MISALIGNED;

    const TwoPass tp = workspace != nullptr
                           ? twopass_kind(T, d_k, d_v, alpha_kind, b_kind, w_kind, dtype)
                           : TP_NONE;
    if (tp != TP_NONE) {
        if (workspace_bytes < twopass_bytes(tp, B, T, H, d_v, b_kind, w_kind)) return GDR_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDR_ERR_MISALIGNED;
    }

    cudaError_t e;
    if (tc_path) {
        if (!encoder()) return GDR_ERR_NO_DEVICE;
        CUtensorMap maps[6];
        // unused maps point at q so every kernel argument is a valid map
        const void* amap = alpha_kind == GDR_GATE_CHANNEL ? alpha : q;
        const void* bmap = b_kind == GDR_GATE_CHANNEL ? b : q;
        const void* wmap = w_kind == GDR_GATE_CHANNEL ? w : q;
        if (!make_map(&maps[0], q, B, T, H_qk, d_k) || !make_map(&maps[1], k, B, T, H_qk, d_k) ||
            !make_map(&maps[2], v, B, T, H, d_v) || !make_map(&maps[3], amap, B, T, H, d_k) ||
            !make_map(&maps[4], bmap, B, T, H, d_k) || !make_map(&maps[5], wmap, B, T, H, d_k))
            return GDR_ERR_INVALID_ARG;
        const bool tied = w_kind == GDR_GATE_TIED && b_kind == GDR_GATE_SCALAR;
        if (tp == TP_GENERAL) {
            e = gdr::launch_chunk_twopass_general(maps, make_map, workspace, q, k, v, alpha, b, w,
                                                  alpha_kind, b_kind, w_kind, S0, o, S_T, d_status,
                                                  B, T, H, d_v, group, allow_segments, st);
        } else if (tp == TP_GDN) {
            CUtensorMap ws_maps[3];
            const uint8_t* pbase = reinterpret_cast<const uint8_t*>(workspace) +
                                   (size_t)B * T * H * d_k * sizeof(uint16_t);
            const uint8_t* aqbase = pbase + (size_t)B * T * H * d_v * sizeof(uint16_t);
            if (!make_map(&ws_maps[0], workspace, B, T, H, d_k) ||
                !make_map(&ws_maps[1], pbase, B, T, H, d_v) || !make_map(&ws_maps[2], aqbase, B, T, H, 64))
                return GDR_ERR_INVALID_ARG;
            e = gdr::launch_chunk_twopass_gdn(maps, ws_maps, workspace, alpha, b, S0, o, S_T,
                                              d_status, B, T, H, d_v, group, st);
        } else if (b_kind == GDR_GATE_NONE)  // no erase: no triangular solve
            e = gdr::launch_chunk_erasefree_sm100(maps, q, k, v, alpha, w, alpha_kind, w_kind, S0, o, S_T,
                                                  d_status, B, T, H, d_v, group, st);
        else
            e = gdr::launch_chunk_sm100(maps, q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, tied, S0, o,
                                        S_T, d_status, B, T, H, d_v, group, st);
    } else if (tp == TP_GDN256) {
        if (!encoder()) return GDR_ERR_NO_DEVICE;
        CUtensorMap maps[3], ws_maps[4];
        const size_t n = (size_t)B * T * H;
        const uint8_t* pbase = reinterpret_cast<const uint8_t*>(workspace) + n * d_k * sizeof(uint16_t);
        const uint8_t* aqbase = pbase + n * d_v * sizeof(uint16_t);
        const uint8_t* ktbase = aqbase + n * 64 * sizeof(uint16_t);
        if (!make_map(&maps[0], q, B, T, H_qk, d_k) || !make_map(&maps[1], k, B, T, H_qk, d_k) ||
            !make_map(&maps[2], v, B, T, H, d_v) || !make_map(&ws_maps[0], workspace, B, T, H, d_k) ||
            !make_map(&ws_maps[1], pbase, B, T, H, d_v) || !make_map(&ws_maps[2], aqbase, B, T, H, 64) ||
            !make_map(&ws_maps[3], ktbase, B, T, H, d_k))
            return GDR_ERR_INVALID_ARG;
        e = gdr::launch_chunk_twopass_gdn256(maps, ws_maps, alpha, b, S0, o, S_T, d_status, B, T, H, d_v,
                                             group, st);
    } else {
        e = gdr::launch_recurrent(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S0, o, S_T, B,
                                  T, H, d_k, d_v, dtype, group, st);
    }
    return e == cudaSuccess ? GDR_OK : GDR_ERR_LAUNCH;
}

}  // namespace gdr

extern "C" {

gdr_status gdr_chunk_fwd_grouped(const void* q, const void* k, const void* v, const void* alpha,
                                 const void* b, const void* w, int alpha_kind, int b_kind,
                                 int w_kind, const float* S0, void* o, float* S_T, void* workspace,
                                 size_t workspace_bytes, int B, int T, int H_qk, int H, int d_k,
                                 int d_v, int chunk, int dtype, int* d_status, void* stream) {
    return gdr::chunk_fwd_impl(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S0, o, S_T,
                               workspace, workspace_bytes, B, T, H_qk, H, d_k, d_v, chunk, dtype,
                               d_status, true, stream);
}

gdr_status gdr_chunk_fwd(const void* q, const void* k, const void* v, const void* alpha,
                         const void* b, const void* w, int alpha_kind, int b_kind, int w_kind,
                         const float* S0, void* o, float* S_T, void* workspace,
                         size_t workspace_bytes, int B, int T, int H, int d_k, int d_v, int chunk,
                         int dtype, int* d_status, void* stream) {
    return gdr_chunk_fwd_grouped(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S0, o, S_T,
                                 workspace, workspace_bytes, B, T, H, H, d_k, d_v, chunk, dtype,
                                 d_status, stream);
}

gdr_status gdr_decode_step_grouped(const void* q, const void* k, const void* v, const void* alpha,
                                   const void* b, const void* w, int alpha_kind, int b_kind,
                                   int w_kind, float* S, void* o, int B, int H_qk, int H, int d_k,
                                   int d_v, int dtype, int* d_status, void* stream) {
    (void)d_status;  // the decode kernel has no bounded waits
    if (B < 1 || H < 1 || d_k < 1 || d_v < 1) return GDR_ERR_INVALID_ARG;
    if (H_qk < 1 || H % H_qk != 0) return GDR_ERR_INVALID_ARG;
    if (dtype != GDR_BF16 && dtype != GDR_FP32) return GDR_ERR_INVALID_ARG;
    if (!kind_ok(alpha_kind, false) || !kind_ok(b_kind, false) || !kind_ok(w_kind, true))
        return GDR_ERR_INVALID_ARG;
    if (!gate_ptr_ok(alpha_kind, alpha) || !gate_ptr_ok(b_kind, b) || !gate_ptr_ok(w_kind, w))
        return GDR_ERR_INVALID_ARG;
    if (w_kind == GDR_GATE_TIED && b_kind == GDR_GATE_NONE) return GDR_ERR_INVALID_ARG;
    if (!q || !k || !v || !S || !o) return GDR_ERR_INVALID_ARG;
    if (d_k > 256 || !(d_v == 16 || d_v == 32 || d_v == 64 || d_v == 128 || d_v == 256) ||
        gdr::decode_rows_per_thread(d_k, d_v) > 32)
        return GDR_ERR_UNSUPPORTED;
    if (!aligned16(S) || !aligned16(o) || !aligned16(q) || !aligned16(k) || !aligned16(v))
        return GDR_ERR_MISALIGNED;
    cudaError_t e = gdr::launch_decode(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S, o, B * H,
                                       d_k, d_v, dtype, H / H_qk, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDR_OK : GDR_ERR_LAUNCH;
}

gdr_status gdr_decode_step(const void* q, const void* k, const void* v, const void* alpha,
                           const void* b, const void* w, int alpha_kind, int b_kind, int w_kind,
                           float* S, void* o, int B, int H, int d_k, int d_v, int dtype,
                           int* d_status, void* stream) {
    return gdr_decode_step_grouped(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S, o, B, H, H,
                                   d_k, d_v, dtype, d_status, stream);
}

}  // extern "C"
