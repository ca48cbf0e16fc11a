// decode_common.cuh -- small device helpers of the CUDA-core decode-step kernels.
#pragma once

#include "common.cuh"

namespace lbca {

template <typename T>
__device__ __forceinline__ void put2(T* p, float a, float b);
template <> __device__ __forceinline__ void put2<float>(float* p, float a, float b) {
    *reinterpret_cast<float2*>(p) = make_float2(a, b);
}
template <> __device__ __forceinline__ void put2<__nv_bfloat16>(__nv_bfloat16* p, float a, float b) {
    *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(a, b);
}
// Two consecutive I/O elements, loaded as raw bits (so that the load can be
// issued early and converted where it is used).
template <typename T> struct Pair;
template <> struct Pair<float> {
    using Raw = float2;
    static __device__ __forceinline__ Raw load(const float* p) { return *reinterpret_cast<const float2*>(p); }
    static __device__ __forceinline__ float2 cvt(Raw r) { return r; }
};
template <> struct Pair<__nv_bfloat16> {
    using Raw = uint32_t;
    static __device__ __forceinline__ Raw load(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }
    static __device__ __forceinline__ float2 cvt(Raw w) {
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
};
template <typename T> __device__ __forceinline__ void unpack16(const uint4& u, float (&o)[Vec<T>::N]);
template <> __device__ __forceinline__ void unpack16<float>(const uint4& u, float (&o)[4]) {
    o[0] = __uint_as_float(u.x); o[1] = __uint_as_float(u.y); o[2] = __uint_as_float(u.z); o[3] = __uint_as_float(u.w);
}
template <> __device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& u, float (&o)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = __uint_as_float(w[i] << 16);
        o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

template <typename T>
__device__ __forceinline__ float2 get2(const T* p) {
    return make_float2(to_f<T>(p[0]), to_f<T>(p[1]));
}

// Online-softmax merge weights of two partials with maxima ma, mb.
__device__ __forceinline__ void merge_weights(float ma, float mb, float& M, float& fa, float& fb) {
    M = fmaxf(ma, mb);
    fa = ma == kNegInf ? 0.f : ex2(ma - M);
    fb = mb == kNegInf ? 0.f : ex2(mb - M);
}

}  // namespace lbca
