// Internal helpers shared by the CUDA translation units of the library.
// Host side: status/error reporting and argument checks. Device side: 16-byte
// vector loads, 16-bit <-> fp32 conversion, and the int8 rounding step.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>
#include <utility>

#include "../../include/sq_api.h"

namespace sq {

// ----------------------------------------------------------------- host side
sq_status_t set_error(sq_status_t st, const char* fmt, ...);
sq_status_t check_launch(const char* what);

inline cudaStream_t as_cuda(sq_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int dtype_bytes(sq_dtype_t dt) {
    switch (dt) {
        case SQ_F32: return 4;
        case SQ_F16: return 2;
        case SQ_BF16: return 2;
        case SQ_I32: return 4;
        case SQ_I8: return 1;
    }
    return 0;
}

int num_sms();  // SM count of the current device (cached per device)

// Kernels are launched with programmatic stream serialisation: a kernel may
// start (and run its prologue) while the previous kernel in the stream is
// finishing. Every kernel executes pdl_wait() before it touches global memory,
// which blocks until the previous grid has completed and its writes are
// visible, so stream order is kept. SQ_DISABLE_PDL=1 turns this off.
bool pdl_enabled();

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same with thread-block clusters of cluster_x CTAs along x (grid.x a
// multiple of cluster_x).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                               int cluster_x, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster_x;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

#define SQ_REQUIRE(cond, status, ...) \
    do {                              \
        if (!(cond)) return ::sq::set_error(status, __VA_ARGS__); \
    } while (0)

// ---------------------------------------------------------------- device side
// Wait for the previous grid in the stream (no-op without a programmatic
// launch), then allow the next one to begin launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Element count of one 16-byte vector.
template <typename T> struct Vec;
template <> struct Vec<__half> { static constexpr int N = 8; };
template <> struct Vec<__nv_bfloat16> { static constexpr int N = 8; };
template <> struct Vec<float> { static constexpr int N = 4; };

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint4 ldg_v4(const void* p) {
    return *reinterpret_cast<const uint4*>(p);
}

// Unpack a 16-byte vector into fp32 (exact for 16-bit sources).
template <typename T>
__device__ __forceinline__ void unpack(const uint4& r, float* f);

template <>
__device__ __forceinline__ void unpack<__nv_bfloat16>(const uint4& r, float* f) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

template <>
__device__ __forceinline__ void unpack<__half>(const uint4& r, float* f) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
        float2 v = __half22float2(h);
        f[2 * i] = v.x;
        f[2 * i + 1] = v.y;
    }
}

template <>
__device__ __forceinline__ void unpack<float>(const uint4& r, float* f) {
    f[0] = __uint_as_float(r.x);
    f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z);
    f[3] = __uint_as_float(r.w);
}

// fp32 -> 16-bit, round to nearest even.
template <typename T> __device__ __forceinline__ uint16_t to16(float v);
template <> __device__ __forceinline__ uint16_t to16<__nv_bfloat16>(float v) {
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t*>(&b);
}
template <> __device__ __forceinline__ uint16_t to16<__half>(float v) {
    __half h = __float2half_rn(v);
    return *reinterpret_cast<uint16_t*>(&h);
}

// int8 code of t: clip to [-127, 127], then round half to even. Clipping
// first gives the same code as rounding first (127.5 -> 127 either way) and
// keeps |t| small enough for the 1.5 * 2^23 shifter: in [2^23, 2^24) fp32
// values are consecutive integers, so one RN add rounds t to an integer
// (ties to even, because the shifter is even) and the low bits hold it.
__device__ __forceinline__ int quant_code(float t) {
    t = fminf(fmaxf(t, -127.0f), 127.0f);
    float r = __fadd_rn(t, 12582912.0f);
    return __float_as_int(r) - 0x4B400000;
}

// Same code without the clip, for a scale taken from the group's own absmax:
// then |t| <= 127 (1 + 2^-23), which rounds to at most 127. Returns the
// shifter's bit pattern; its low byte is the code (the shifter's low byte is 0).
__device__ __forceinline__ uint32_t quant_bits_noclip(float t) {
    return __float_as_uint(__fadd_rn(t, 12582912.0f));
}
__device__ __forceinline__ uint32_t quant_bits_clip(float t) {
    return __float_as_uint(__fadd_rn(fminf(fmaxf(t, -127.0f), 127.0f), 12582912.0f));
}
// Low bytes of four words into one word (byte i from word i).
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic): each lane is one correctly
// rounded fp32 operation, identical to the scalar __fmul_rn / __fadd_rn.
__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// fma on packed pairs: each lane one fused, correctly rounded fma (the
// scalar __fmaf_rn of that lane)
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
// v[e] *= s[e] for 8 values, two at a time
__device__ __forceinline__ void mul8(float* v, const float* s) {
#pragma unroll
    for (int e = 0; e < 8; e += 2) upk2(mul2(pk2(v[e], v[e + 1]), pk2(s[e], s[e + 1])), v[e], v[e + 1]);
}
// Packed pairs are used only where a product is not followed by an add that
// must see it rounded: a packed multiply feeding a packed add has been seen to
// produce the fused (singly rounded) result, which would change int8 codes at
// exact ties. The int8 step below therefore stays scalar.
__device__ __forceinline__ void quant_bits8_noclip(const float* v, float qs, uint32_t* b) {
#pragma unroll
    for (int e = 0; e < 8; ++e) b[e] = quant_bits_noclip(__fmul_rn(v[e], qs));
}

// max on non-negative floats through their bit patterns (monotone for >= 0).
__device__ __forceinline__ void atomic_max_nonneg(float* addr, float v) {
    atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));
}

__device__ __forceinline__ uint32_t pack4_i8(int a, int b, int c, int d) {
    return (uint32_t(a) & 0xffu) | ((uint32_t(b) & 0xffu) << 8) | ((uint32_t(c) & 0xffu) << 16) |
           ((uint32_t(d) & 0xffu) << 24);
}

}  // namespace sq
