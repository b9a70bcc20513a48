// gdr_chunk_fwd_static: gdr_chunk_fwd with the two-pass path's workspace
// taken from a fixed device array owned by the library instead of the caller.
// The call allocates nothing: the array is a file-scope __device__ object of
// this translation unit, placed in device memory when its module loads; its
// address is looked up once per device and cached.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "gdr.h"

namespace gdr {
gdr_status chunk_fwd_impl(const void* q, const void* k, const void* v, const void* alpha,
                          const void* b, const void* w, int alpha_kind, int b_kind, int w_kind,
                          const float* S0, void* o, float* S_T, void* workspace,
                          size_t workspace_bytes, int B, int T, int H_qk, int H, int d_k, int d_v,
                          int chunk, int dtype, int* d_status, bool allow_segments, void* stream);
}  // namespace gdr

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" {

size_t gdr_chunk_fwd_static_capacity(void) { return kStaticScratchBytes; }

gdr_status gdr_chunk_fwd_static(const void* q, const void* k, const void* v, const void* alpha,
                                const void* b, const void* w, int alpha_kind, int b_kind,
                                int w_kind, const float* S0, void* o, float* S_T, int B, int T,
                                int H, int d_k, int d_v, int chunk, int dtype, int* d_status,
                                void* stream) {
    const size_t need =
        gdr_chunk_fwd_workspace_size(B, T, H, d_k, d_v, alpha_kind, b_kind, w_kind, dtype);
    if (need > kStaticScratchBytes) return GDR_ERR_UNSUPPORTED;
    void* ws = nullptr;
    if (need > 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
            return GDR_ERR_NO_DEVICE;
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_scratch_addr[dev] &&
            cudaGetSymbolAddress(&g_scratch_addr[dev], g_static_scratch) != cudaSuccess) {
            g_scratch_addr[dev] = nullptr;
            return GDR_ERR_LAUNCH;
        }
        ws = g_scratch_addr[dev];
    }
    // no auxiliary stream or events: this call creates no CUDA objects either
    return gdr::chunk_fwd_impl(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S0, o, S_T, ws,
                               need, B, T, H, H, d_k, d_v, chunk, dtype, d_status, false, stream);
}

}  // extern "C"
