// Pieces shared by the chunkwise tensor-core kernels: sizes, launch
// parameters, and bf16 packing helpers for 128-byte-swizzled tiles.
#pragma once

#include "common.cuh"

namespace gdr {
namespace chunkc {

constexpr int C = 64;     // chunk length
constexpr int DK = 128;   // key dimension
constexpr int NV = 64;    // value columns per CTA
constexpr int NT = 256;   // threads per CTA (two warpgroups)

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

__device__ __forceinline__ void st_chunk(uint8_t* base, uint32_t off, const float* x8) {
    uint4 u;
    u.x = pack_bf16x2(x8[0], x8[1]);
    u.y = pack_bf16x2(x8[2], x8[3]);
    u.z = pack_bf16x2(x8[4], x8[5]);
    u.w = pack_bf16x2(x8[6], x8[7]);
    *reinterpret_cast<uint4*>(base + off) = u;
}

__device__ __forceinline__ void st_zero_chunk(uint8_t* base, uint32_t off) {
    *reinterpret_cast<uint4*>(base + off) = make_uint4(0u, 0u, 0u, 0u);
}

// Four bf16 channels [4 cg, 4 cg + 4) of row r of a swizzled 128-column tile.
__device__ __forceinline__ uint32_t piece4(int r, int cg, int rows) {
    return sw128_chunk(r, cg >> 1, rows) + (uint32_t)(cg & 1) * 8u;
}

__device__ __forceinline__ void ld4(const uint8_t* base, uint32_t off, float* x4) {
    const uint2 u = *reinterpret_cast<const uint2*>(base + off);
    const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    x4[0] = f0.x; x4[1] = f0.y; x4[2] = f1.x; x4[3] = f1.y;
}

__device__ __forceinline__ void st4(uint8_t* base, uint32_t off, const float* x4) {
    uint2 u;
    u.x = pack_bf16x2(x4[0], x4[1]);
    u.y = pack_bf16x2(x4[2], x4[3]);
    *reinterpret_cast<uint2*>(base + off) = u;
}

}  // namespace chunkc
}  // namespace gdr
