// common.cuh -- helpers shared by the sm_100a kernels of libdit_block.so:
// 128-bit streaming loads and stores, bf16x8 <-> fp32 conversion, warp
// reductions, per-device attribute cache and host-side argument checks.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "dit_block.h"

namespace dit {

// ------------------------------------------------------------ memory ops

// Read-once data: non-coherent path, no L1 allocation.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Write-once data: streaming store.
__device__ __forceinline__ void st_stream(uint4* p, const uint4& v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// 256-bit forms (sm_100): 32-byte aligned, eight 32-bit words.  Loads are
// evict-first with a 256-byte L2 fetch hint (whole DRAM bursts).
struct alignas(32) u32x8 {
    uint32_t w[8];
};

__device__ __forceinline__ u32x8 ld_stream256(const void* p) {
    u32x8 v;
    asm volatile(
        "ld.global.nc.L1::no_allocate.L2::evict_first.L2::256B.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, "
        "[%8];"
        : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]), "=r"(v.w[5]),
          "=r"(v.w[6]), "=r"(v.w[7])
        : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream256(void* p, const u32x8& v) {
    asm volatile("st.global.cs.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v.w[0]),
                 "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]), "r"(v.w[6]),
                 "r"(v.w[7])
                 : "memory");
}

inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// In-place data (read then written by the same thread): a plain coherent
// load that still skips L1.
__device__ __forceinline__ uint4 ld_inplace(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// In-place data, 32 bytes: coherent, skips L1, evict-first in L2.
__device__ __forceinline__ u32x8 ld_inplace256(const void* p) {
    u32x8 v;
    asm volatile(
        "ld.global.L1::no_allocate.L2::evict_first.L2::256B.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, "
        "[%8];"
        : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]), "=r"(v.w[5]),
          "=r"(v.w[6]), "=r"(v.w[7])
        : "l"(p));
    return v;
}

// ------------------------------------------------------ bf16 conversion

// bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 word.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// Two fp32 -> packed bf16x2, round to nearest even (lo in the low half).
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    uint4 v;
    v.x = pack2(f[0], f[1]);
    v.y = pack2(f[2], f[3]);
    v.z = pack2(f[4], f[5]);
    v.w = pack2(f[6], f[7]);
    return v;
}

// ---------------------------------------------------------- reductions

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ------------------------------------------------------------ host side

// SM count of the current device (cached per device, thread-safe).
int device_sm_count();

// Resident CTAs per SM for a kernel at a block size and dynamic smem
// (cached per device and kernel).
int occupancy(const void* kernel, int threads, size_t smem);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// [a, a + na) and [b, b + nb) in bytes intersect.
inline bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return na && nb && x < y + nb && y < x + na;
}

inline int launch_status() {
    return cudaGetLastError() == cudaSuccess ? DIT_OK : DIT_ERR_LAUNCH;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace dit
