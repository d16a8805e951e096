// Shared host/device helpers of libqknorm: error reporting, alignment checks,
// bf16 <-> fp32 conversion of 16-byte chunks, and streaming memory accesses.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qknorm.h"

namespace qkn {

// Thread-local message behind qkn_last_error(); returns `st` for chaining.
qkn_status fail(qkn_status st, const char *fmt, ...);

// Maps a CUDA runtime error to QKN_ERR_CUDA with the runtime's message.
qkn_status cuda_fail(cudaError_t e, const char *what);

// Checks the launch(es) just issued; QKN_OK when the runtime reports none.
qkn_status check_launch(const char *what);

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline size_t dtype_size(qkn_dtype t) { return t == QKN_F32 ? 4 : 2; }

inline bool valid_dtype(int t) { return t == QKN_F32 || t == QKN_BF16; }

// n_seg within [1, QKN_MAX_SEG], else QKN_ERR_SHAPE with a message.
inline qkn_status check_seg(int n_seg) {
    if (n_seg < 1 || n_seg > QKN_MAX_SEG) return fail(QKN_ERR_SHAPE, "n_seg=%d outside [1, %d]", n_seg, QKN_MAX_SEG);
    return QKN_OK;
}

// Number of SMs of the current device (cached per device).
int sm_count();

// Reads the norm kernels' device error word into *flag and clears it.
qkn_status read_norm_error(int *flag);

// ---------------------------------------------------------------- device side

// Streaming 16-byte load: data read once, evict-first in L1 and L2.
__device__ __forceinline__ uint4 ld_stream(const void *p) {
    return __ldcs(reinterpret_cast<const uint4 *>(p));
}

// Streaming 16-byte store.  Volatile asm keeps stores in program order with
// the other volatile accesses below, which bounds register pressure.
__device__ __forceinline__ void st_stream(void *p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w) : "memory");
}

// Cached read-only 16- and 8-byte loads kept in program order (see st_stream).
__device__ __forceinline__ uint4 ld_ro_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ uint2 ld_ro_v2(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

// bf16 bit pattern (low / high half of a 32-bit word) -> fp32, exact.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two fp32 -> packed bf16x2 with round-to-nearest-even (lo in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// A 16-byte chunk of activations of type T as fp32 values.
template <typename T> struct Chunk;

template <> struct Chunk<float> {
    static constexpr int E = 4;
    __device__ __forceinline__ static void unpack(const uint4 &v, float (&f)[E]) {
        f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
    }
    __device__ __forceinline__ static void unpack_again(const uint4 &v, float (&f)[E]) { unpack(v, f); }
    __device__ __forceinline__ static uint4 pack(const float (&f)[E]) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                          __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};

template <> struct Chunk<__nv_bfloat16> {
    static constexpr int E = 8;
    __device__ __forceinline__ static void unpack(const uint4 &v, float (&f)[E]) {
        f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
        f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
    }
    // Same values as unpack(), formed with byte permutes: a second unpack of a
    // chunk is then recomputed rather than kept live from the first one.
    __device__ __forceinline__ static void unpack_again(const uint4 &v, float (&f)[E]) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(__byte_perm(w[i], 0u, 0x1044u));
            f[2 * i + 1] = __uint_as_float(__byte_perm(w[i], 0u, 0x3244u));
        }
    }
    __device__ __forceinline__ static uint4 pack(const float (&f)[E]) {
        return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                          pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
    }
};

// Loads E consecutive weights of type TW (read-only path, cached) as fp32.
template <typename TW, int E>
__device__ __forceinline__ void load_weights(const TW *w, float (&f)[E]);

template <>
__device__ __forceinline__ void load_weights<float, 4>(const float *w, float (&f)[4]) {
    Chunk<float>::unpack(ld_ro_v4(w), f);
}
template <>
__device__ __forceinline__ void load_weights<float, 8>(const float *w, float (&f)[8]) {
    uint4 a = ld_ro_v4(w), b = ld_ro_v4(w + 4);
    f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y); f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
    f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y); f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
}
template <>
__device__ __forceinline__ void load_weights<__nv_bfloat16, 8>(const __nv_bfloat16 *w, float (&f)[8]) {
    Chunk<__nv_bfloat16>::unpack(ld_ro_v4(w), f);
}
template <>
__device__ __forceinline__ void load_weights<__nv_bfloat16, 4>(const __nv_bfloat16 *w, float (&f)[4]) {
    uint2 a = ld_ro_v2(w);
    f[0] = bf16lo(a.x); f[1] = bf16hi(a.x); f[2] = bf16lo(a.y); f[3] = bf16hi(a.y);
}

// Same values as load_weights, through plain read-only-path intrinsics that
// the compiler may batch and hoist (for kernels with registers to spare).
template <typename TW, int E>
__device__ __forceinline__ void load_weights_batched(const TW *w, float (&f)[E]) {
    if constexpr (sizeof(TW) * E == 16) {
        const uint4 a = __ldg(reinterpret_cast<const uint4 *>(w));
        if constexpr (E == 8) {
            Chunk<__nv_bfloat16>::unpack(a, f);
        } else {
            Chunk<float>::unpack(a, f);
        }
    } else if constexpr (sizeof(TW) * E == 32) {
        const uint4 a = __ldg(reinterpret_cast<const uint4 *>(w));
        const uint4 b = __ldg(reinterpret_cast<const uint4 *>(w) + 1);
        f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y); f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
        f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y); f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
    } else {
        const uint2 a = __ldg(reinterpret_cast<const uint2 *>(w));
        f[0] = bf16lo(a.x); f[1] = bf16hi(a.x); f[2] = bf16lo(a.y); f[3] = bf16hi(a.y);
    }
}

// Streaming 16-byte store through the intrinsic (freely schedulable).
__device__ __forceinline__ void st_stream_batched(void *p, uint4 v) {
    __stcs(reinterpret_cast<uint4 *>(p), v);
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

}  // namespace qkn
