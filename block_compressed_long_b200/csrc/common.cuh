// common.cuh -- device helpers shared by the block-compressed attention kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lbca.h"

namespace lbca {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kNegInf = -__builtin_huge_valf();

// 2^x on the SFU (PTX ex2.approx, relative error ~2^-22); all softmax
// exponentials run in the log2 domain with log2(e) folded into the logits.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- 16-byte vectors of I/O elements, widened to f32 ---------------------------
template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int N = 4; };
template <> struct Vec<__nv_bfloat16> { static constexpr int N = 8; };

__device__ __forceinline__ void ld16(const float* p, float (&o)[4]) {
    float4 v = *reinterpret_cast<const float4*>(p);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void ld16(const __nv_bfloat16* p, float (&o)[8]) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = __uint_as_float(w[i] << 16);
        o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
// Streaming (L1-bypassing) variants for data read once.
__device__ __forceinline__ void ld16_cs(const float* p, float (&o)[4]) {
    float4 v = __ldcs(reinterpret_cast<const float4*>(p));
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void ld16_cs(const __nv_bfloat16* p, float (&o)[8]) {
    uint4 v = __ldcs(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = __uint_as_float(w[i] << 16);
        o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
// 8 floats -> 8 fp16 (16 bytes)
__device__ __forceinline__ void st16_f16(__half* p, const float (&o)[8]) {
    uint4 v;
    v.x = pack_f16x2(o[0], o[1]);
    v.y = pack_f16x2(o[2], o[3]);
    v.z = pack_f16x2(o[4], o[5]);
    v.w = pack_f16x2(o[6], o[7]);
    *reinterpret_cast<uint4*>(p) = v;
}
// The same, flagging any value beyond the fp16 range (it would become inf).
__device__ __forceinline__ void st16_f16_checked(__half* p, const float (&o)[8], bool& ovf) {
#pragma unroll
    for (int i = 0; i < 8; ++i) ovf |= fabsf(o[i]) > 65504.f;
    st16_f16(p, o);
}
__device__ __forceinline__ void st16(float* p, const float (&o)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
}
__device__ __forceinline__ void st16(__nv_bfloat16* p, const float (&o)[8]) {
    uint4 v;
    v.x = pack_bf16x2(o[0], o[1]);
    v.y = pack_bf16x2(o[2], o[3]);
    v.z = pack_bf16x2(o[4], o[5]);
    v.w = pack_bf16x2(o[6], o[7]);
    *reinterpret_cast<uint4*>(p) = v;
}

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// ---- RoPE -------------------------------------------------------------------------
// Pair k (dims D - rho + 2k, +1) turns by pos * inv_k radians per position,
// inv_k = theta^(-2k/rho) = step^k with step = theta^(-2/rho) computed in fp64 on
// the host.  Positions reach 1e5+, where an fp32 product pos * inv_k would be
// off by milliradians, so the angle is formed in turns in 64-bit fixed point:
// F_k = inv_k / (2 pi) * 2^64 and pos * F_k wraps exactly modulo one turn (two's
// complement makes negative positions come out right too).  The top 24 bits of
// the fraction (2^-24 turn resolution) then go to sincospif on [0, 2).
// F_k of pair k (fixed-point turns per position): step^k / (2 pi) * 2^64, with
// step^k by repeated squaring in fp64.  Host and device compute it alike.
__host__ __device__ __forceinline__ uint64_t rope_turns(int k, double step) {
    double inv = 1.0, b = step;
    for (int e = k; e; e >>= 1) {
        if (e & 1) inv *= b;
        b *= b;
    }
    const double kTurn = 0.15915494309189535;            // 1 / (2 pi)
    const double kTwo64 = 18446744073709551616.0;        // 2^64
    return (uint64_t)(inv * kTurn * kTwo64);
}
// cos / sin of position pos on the pair whose turns per position are F.
__device__ __forceinline__ float2 rope_cs_turns(int64_t pos, uint64_t F) {
    const uint64_t t = (uint64_t)pos * F;
    const float x = (float)(uint32_t)(t >> 40) * (1.0f / 16777216.0f);
    float sn, cs;
    sincospif(2.0f * x, &sn, &cs);
    return make_float2(cs, sn);
}
__device__ __forceinline__ float2 rope_cs(int64_t pos, int k, double step) {
    return rope_cs_turns(pos, rope_turns(k, step));
}
// (x, y) turned by the angle whose cosine and sine are cs.  Spelt out as one
// rounded product and one fused multiply-add per component so that every
// kernel rounds a rotation identically (the compiler may not contract it
// differently from one kernel to the next).
__device__ __forceinline__ void rotate_pair(float& a, float& b, float2 cs) {
    const float x = a, y = b;
    a = __fmaf_rn(x, cs.x, -__fmul_rn(y, cs.y));
    b = __fmaf_rn(x, cs.y, __fmul_rn(y, cs.x));
}

// ---- programmatic dependent launch --------------------------------------------------
// Launched with programmatic stream serialisation, a kernel may start while the
// preceding kernel on its stream drains: work before griddep_wait() must not
// read what that kernel writes.  Without the launch attribute both are no-ops.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- status -------------------------------------------------------------------------
__device__ __forceinline__ void set_status(int32_t* st, int32_t code) {
    if (st) atomicCAS(st, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarrier + bulk async copy (the non-tensor TMA path) -------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}
// Global -> shared bulk copy completing on `bar`.  dst, src 16-byte aligned,
// bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: gives up after `limit_ns` of wall time and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          uint64_t limit_ns = 200ull * 1000 * 1000) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// Rows [r, r + n) of an array of `rows` rows.  In the bounds-checked build
// (LBCA_CHECKED) a range that leaves the array records LBCA_ERR_ARG on the
// status word and is moved to the array's start, so the access stays inside
// it (the result is then wrong, and flagged); otherwise r is returned as is.
__device__ __forceinline__ long long checked_rows(long long r, long long n, long long rows, int32_t* status) {
#ifdef LBCA_CHECKED
    if (r < 0 || n < 0 || r + n > rows) {
        set_status(status, LBCA_ERR_ARG);
        return 0;
    }
#else
    (void)n; (void)rows; (void)status;
#endif
    return r;
}

// The current device ordinal, or -1 (beyond 64 devices, or no device): kernel
// attributes are set once per device, since a process may drive several.
inline int current_device() {
    int d = 0;
    return cudaGetDevice(&d) == cudaSuccess && d >= 0 && d < 64 ? d : -1;
}

__device__ __forceinline__ int visible_blocks(int L, int m, int w) {
    int p = L - w;
    return p > 0 ? p / m : 0;
}

}  // namespace lbca
