// Shared device helpers for the HiKVP kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace akv {

// Device status word values (sticky; first error wins).
enum : int { kDevOk = 0, kDevBadChild = 1, kDevTimeout = 2, kDevBadSmem = 3 };

// Programmatic dependent launch.  griddep_wait: wait until the grid this one
// depends on (the previous kernel on the stream, when this one was launched
// with programmatic stream serialization) has completed and its writes are
// visible; a no-op otherwise.  griddep_launch: allow the next grid on the
// stream to start launching (its CTAs then wait in griddep_wait).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void set_status(int *status, int code)
{
    atomicCAS(status, kDevOk, code);
}

// Raw binary32 bits of a stored element (bfloat16 widens exactly).
__device__ __forceinline__ uint32_t elem_bits(float x) { return __float_as_uint(x); }
__device__ __forceinline__ uint32_t elem_bits(__nv_bfloat16 x)
{
    return ((uint32_t)__bfloat16_as_ushort(x)) << 16;
}
__device__ __forceinline__ float elem_f32(float x) { return x; }
__device__ __forceinline__ float elem_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Unpack the 16-byte vector `v` into E floats (E = 8 for bfloat16, 4 for float).
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int E = 8;
    __device__ __forceinline__ static void unpack(const uint4 &v, float *o)
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};
template <> struct Vec16<float> {
    static constexpr int E = 4;
    __device__ __forceinline__ static void unpack(const uint4 &v, float *o)
    {
        o[0] = __uint_as_float(v.x);
        o[1] = __uint_as_float(v.y);
        o[2] = __uint_as_float(v.z);
        o[3] = __uint_as_float(v.w);
    }
};

__device__ __forceinline__ uint4 ldg16(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// Order-preserving map of a float to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f)
{
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k)
{
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

}  // namespace akv
