// device_common.cuh -- device helpers of the walk kernels: bf16 bit handling,
// 16-byte vector access to feature rows, the cp.async copies of the
// shared-memory rings and exact dot products.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#ifndef AG_RING_L1
#define AG_RING_L1 0      // 1: ring copies also allocate in L1 (cp.async.ca), 0: L2 only (.cg)
#endif

namespace ag {
namespace {

using bf16_t = uint16_t;  // bfloat16 stored as raw bits

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
__device__ __forceinline__ uint32_t bf16_bits(float f) {
    return uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) { return bf16_bits(a) | (bf16_bits(b) << 16); }

// Vector access to VEC consecutive features: gathered rows stay in their
// storage type ("raw") until they are used, so that several rows in flight
// cost only their own size in registers.
template <typename T, int VEC> struct Vec;

template <> struct Vec<float, 4> {
    using raw = float4;
    static __device__ __forceinline__ raw zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
    static __device__ __forceinline__ raw load_raw(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
    static __device__ __forceinline__ void unpack(raw t, float (&v)[4]) { v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w; }
    static __device__ __forceinline__ void store(float *p, const float (&v)[4]) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
    }
};
template <> struct Vec<float, 1> {
    using raw = float;
    static __device__ __forceinline__ raw zero() { return 0.f; }
    static __device__ __forceinline__ raw load_raw(const float *p) { return __ldg(p); }
    static __device__ __forceinline__ void unpack(raw t, float (&v)[1]) { v[0] = t; }
    static __device__ __forceinline__ void store(float *p, const float (&v)[1]) { __stcs(p, v[0]); }
};
template <> struct Vec<bf16_t, 8> {
    using raw = uint4;
    static __device__ __forceinline__ raw zero() { return make_uint4(0u, 0u, 0u, 0u); }
    static __device__ __forceinline__ raw load_raw(const bf16_t *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }
    static __device__ __forceinline__ void unpack(raw t, float (&v)[8]) {
        v[0] = bf16_lo(t.x); v[1] = bf16_hi(t.x); v[2] = bf16_lo(t.y); v[3] = bf16_hi(t.y);
        v[4] = bf16_lo(t.z); v[5] = bf16_hi(t.z); v[6] = bf16_lo(t.w); v[7] = bf16_hi(t.w);
    }
    static __device__ __forceinline__ void store(bf16_t *p, const float (&v)[8]) {
        uint4 t = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                             pack_bf16(v[6], v[7]));
        __stcs(reinterpret_cast<uint4 *>(p), t);
    }
};
template <> struct Vec<bf16_t, 2> {
    using raw = uint32_t;
    static __device__ __forceinline__ raw zero() { return 0u; }
    static __device__ __forceinline__ raw load_raw(const bf16_t *p) {
        return __ldg(reinterpret_cast<const unsigned int *>(p));
    }
    static __device__ __forceinline__ void unpack(raw t, float (&v)[2]) { v[0] = bf16_lo(t); v[1] = bf16_hi(t); }
    static __device__ __forceinline__ void store(bf16_t *p, const float (&v)[2]) {
        __stcs(reinterpret_cast<unsigned int *>(p), pack_bf16(v[0], v[1]));
    }
};
template <> struct Vec<bf16_t, 1> {
    using raw = uint32_t;
    static __device__ __forceinline__ raw zero() { return 0u; }
    static __device__ __forceinline__ raw load_raw(const bf16_t *p) {
        return uint32_t(__ldg(reinterpret_cast<const unsigned short *>(p)));
    }
    static __device__ __forceinline__ void unpack(raw t, float (&v)[1]) { v[0] = __uint_as_float(t << 16); }
    static __device__ __forceinline__ void store(bf16_t *p, const float (&v)[1]) {
        *reinterpret_cast<unsigned short *>(p) = (unsigned short)bf16_bits(v[0]);
    }
};

template <typename T, int VEC>
__device__ __forceinline__ void load_vec(const T *p, float (&v)[VEC]) {
    Vec<T, VEC>::unpack(Vec<T, VEC>::load_raw(p), v);
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
#if AG_RING_L1
    asm volatile("cp.async.ca.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
#else
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
#endif
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// dot product of two raw 16-byte vectors, accumulated in order into c.
// bf16: fma.rn.f32.bf16 multiplies two bf16 values exactly and adds in fp32
// with one rounding -- the same result as widening both to fp32 first.
__device__ __forceinline__ float dot_raw(float4 a, float4 b, float c) {
    c = fmaf(a.x, b.x, c);
    c = fmaf(a.y, b.y, c);
    c = fmaf(a.z, b.z, c);
    return fmaf(a.w, b.w, c);
}
__device__ __forceinline__ float dot2_bf16(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\t"
        "mov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %3;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
        : "=f"(d)
        : "r"(a), "r"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float dot_raw(uint4 a, uint4 b, float c) {
    c = dot2_bf16(a.x, b.x, c);
    c = dot2_bf16(a.y, b.y, c);
    c = dot2_bf16(a.z, b.z, c);
    return dot2_bf16(a.w, b.w, c);
}

}  // namespace
}  // namespace ag
