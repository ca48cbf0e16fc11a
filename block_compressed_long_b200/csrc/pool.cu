// pool.cu -- block pooling, raw-window fill and streaming append.
//
// Block pooling (HCA page, "What is implemented", Eqs 20-23: one series, the
// m tokens of a block folded into one entry by softmax weights computed from
// their content plus a learned bias per position in the block; mSeek README,
// "How LBCA works", steps 2-3):
// per (block j, kv head g, channel c) the weights are softmax_i(Z + B_pos[i])
// over the block's m positions and the entry is the weighted sum of X.  Key
// entries are then finalised: RMSNorm (HCA form) and RoPE at the block-start
// position (CSA page, "Deviations from paper").
//
// B200 mapping: HBM-bound streaming.  One CTA per (block, sequence); each
// thread owns one 16-byte vector of channels (8 bf16 / 4 f32) of the G*D row,
// so every token row is read with fully coalesced 128-bit streaming loads.
// The per-channel softmax runs online in registers, four tokens per step with
// the loads of a step issued together, one rescale per step and base-2
// exponentials on the SFU.  Registers are kept low enough that a whole launch
// of the common shapes is resident at once (memory parallelism from warps).  RMSNorm needs a per-head reduction, done
// deterministically through shared memory.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace lbca {
namespace {

template <typename T> __device__ __forceinline__ void unpack(const uint4& u, float (&o)[Vec<T>::N]);
template <> __device__ __forceinline__ void unpack<float>(const uint4& u, float (&o)[4]) {
    o[0] = __uint_as_float(u.x); o[1] = __uint_as_float(u.y);
    o[2] = __uint_as_float(u.z); o[3] = __uint_as_float(u.w);
}
template <> __device__ __forceinline__ void unpack<__nv_bfloat16>(const uint4& u, float (&o)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = __uint_as_float(w[i] << 16);
        o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// Sum of `v` over the `nvh` consecutive threads starting at `first` (one kv
// head's vectors).  Deterministic order; every thread of the CTA must call it.
__device__ __forceinline__ float head_sum(float* part, float v, int first, int nvh) {
    part[threadIdx.x] = v;
    __syncthreads();
    float s = 0.f;
    for (int i = 0; i < nvh; ++i) s += part[first + i];
    __syncthreads();
    return s;
}

// RMSNorm scale and gain, then RoPE of the pairs that fall in the rotated dims.
template <typename T, int VEC>
__device__ __forceinline__ void finalise_key(float (&e)[VEC], int d0, int D, bool rms, float ss,
                                             float eps, const T* gamma, int rho, const float2* cs) {
    if (rms) {
        const float inv = 1.0f / sqrtf(ss / (float)D + eps);
#pragma unroll
        for (int i = 0; i < VEC; ++i) e[i] *= inv * (gamma ? to_f<T>(gamma[d0 + i]) : 1.0f);
    }
    if (rho) {
        const int base = D - rho;
#pragma unroll
        for (int i = 0; i < VEC; i += 2) {
            const int d = d0 + i;
            if (d >= base) rotate_pair(e[i], e[i + 1], cs[(d - base) >> 1]);
        }
    }
}

// CTA = (block j, sequence b, slice of whole kv heads, series); <= 256
// threads.  RAW: also the fp16 copy of every token of a complete block (the
// tensor-core prefill's operands), in an instantiation of its own so that
// plain pooling carries none of it.  DUAL: dual overlapped pooling (CSA page,
// "What is implemented", Eqs 9-12): entry j folds block j - 1 of the b-series
// (none for j = 0) and then block j of the a-series into one online softmax.
template <typename T, bool RAW, bool DUAL>
__global__ void __launch_bounds__(256, 2) pool_kernel(const PoolArgs a) {
    constexpr int VEC = Vec<T>::N;
    constexpr int U = 4;  // tokens per online-softmax step
    extern __shared__ __align__(16) float smem[];
    const PoolSeries& sr = a.ser[blockIdx.z / a.gz];
    const int GD = a.G * a.D, NVH = a.D / VEC;
    const int hpc = blockDim.x / NVH;  // heads per CTA
    const int hs = blockIdx.z % a.gz;
    const int j = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const bool active = tid < hpc * NVH && hs * hpc + tid / NVH < a.G;
    const int cv = active ? hs * hpc * NVH + tid : 0;  // vector index within the G*D row
    const int n_tok = min(a.m, a.T - j * a.m);
    const bool full = n_tok == a.m;
    float2* cs = reinterpret_cast<float2*>(smem);
    float* part = smem + a.rho;
    if (full && sr.key && a.rho)
        for (int k = tid; k < a.rho / 2; k += blockDim.x)
            cs[k] = rope_cs(a.pos0 + (int64_t)j * a.m, k, a.rope_step);
    __syncthreads();

    const int rstride = GD / VEC;  // uint4 per token row
    float mx[VEC], l[VEC], acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) { mx[e] = kNegInf; l[e] = 0.f; acc[e] = 0.f; }
    const int g = cv / NVH, d0 = (cv % NVH) * VEC;
    bool f16_ovf = false;  // an fp16 copy left the fp16 range

    // Fold the n tokens of one block of one series (raw rows from xs, zs, the
    // bias rows from bs) into the running softmax.  U tokens per step: their
    // X, Z and B_pos vectors are loaded together (12 x 16 bytes in flight per
    // thread), then one rescale and U accumulations.  Memory parallelism comes
    // from many resident warps (few registers per thread).
    auto fold = [&](const uint4* xp, const uint4* zp, const uint4* bp, int n, int blk, bool raw_copy) {
        for (int i0 = 0; i0 < n; i0 += U) {
            uint4 cx[U], cz[U], cb[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (i0 + u < n) {
                    cx[u] = __ldcs(xp + (size_t)(i0 + u) * rstride);
                    cz[u] = __ldcs(zp + (size_t)(i0 + u) * rstride);
                    cb[u] = __ldg(bp + (size_t)(i0 + u) * rstride);
                }
            if constexpr (RAW && !DUAL && VEC == 8) {
                if (raw_copy) {  // these tokens' fp16 copy; keys turned at their position
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        if (i0 + u < n) {
                            float xf[VEC];
                            unpack<T>(cx[u], xf);
                            const int s_tok = blk * a.m + i0 + u;
                            const int dr = d0 - (a.D - a.rho);
                            if (sr.key && a.rho)
#pragma unroll
                                for (int e = 0; e < VEC; e += 2)
                                    if (dr + e >= 0)
                                        rotate_pair(xf[e], xf[e + 1], a.tab[(size_t)((dr + e) >> 1) * a.T + s_tok]);
                            st16_f16_checked(static_cast<__half*>(sr.raw_f16) +
                                                 ((size_t)b * a.T + s_tok) * GD + (size_t)cv * VEC,
                                             xf, f16_ovf);
                        }
                }
            }
            float cmax[VEC];
#pragma unroll
            for (int e = 0; e < VEC; ++e) cmax[e] = mx[e];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (i0 + u < n) {
                    float zf[VEC], bf[VEC];
                    unpack<T>(cz[u], zf);
                    unpack<T>(cb[u], bf);
#pragma unroll
                    for (int e = 0; e < VEC; ++e) cmax[e] = fmaxf(cmax[e], (zf[e] + bf[e]) * kLog2e);
                }
            }
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                const float r = ex2(mx[e] - cmax[e]);
                l[e] *= r;
                acc[e] *= r;
                mx[e] = cmax[e];
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (i0 + u < n) {
                    float xf[VEC], zf[VEC], bf[VEC];
                    unpack<T>(cx[u], xf);
                    unpack<T>(cz[u], zf);
                    unpack<T>(cb[u], bf);
#pragma unroll
                    for (int e = 0; e < VEC; ++e) {
                        const float p = ex2((zf[e] + bf[e]) * kLog2e - mx[e]);
                        l[e] += p;
                        acc[e] = fmaf(p, xf[e], acc[e]);
                    }
                }
            }
        }
    };
    auto series_rows = [&](const void* x, int blk) {
        return reinterpret_cast<const uint4*>(static_cast<const T*>(x) + ((size_t)b * a.T + (size_t)blk * a.m) * GD +
                                              (size_t)cv * VEC);
    };
    if (active) {
        if constexpr (DUAL) {
            if (j > 0)  // the preceding block of the b-series joins the same softmax
                fold(series_rows(sr.xb, j - 1), series_rows(sr.zb, j - 1),
                     reinterpret_cast<const uint4*>(static_cast<const T*>(sr.bposb) + (size_t)cv * VEC), a.m, j - 1,
                     false);
        }
        fold(series_rows(sr.x, j), series_rows(sr.z, j),
             reinterpret_cast<const uint4*>(static_cast<const T*>(sr.bpos) + (size_t)cv * VEC), n_tok, j,
             full && sr.raw_f16 != nullptr);
    }

    if (full) {
        float e[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) e[i] = active ? acc[i] / l[i] : 0.f;
        float ss = 0.f;
        if (sr.key && a.rmsnorm) {
            float v = 0.f;
#pragma unroll
            for (int i = 0; i < VEC; ++i) v += e[i] * e[i];
            ss = head_sum(part, v, active ? tid - (cv % NVH) : 0, NVH);
        }
        if (sr.key)
            finalise_key<T, VEC>(e, d0, a.D, a.rmsnorm, ss, a.eps, static_cast<const T*>(sr.gamma), a.rho, cs);
        if (active) {
            const size_t oi = (((size_t)b * a.G + g) * a.out_blocks + a.blk_off + j) * a.D + d0;
            if (sr.out) st16(static_cast<T*>(sr.out) + oi, e);
            if (sr.out_f32) {
#pragma unroll
                for (int i = 0; i < VEC; i += 4)
                    *reinterpret_cast<float4*>(sr.out_f32 + oi + i) = make_float4(e[i], e[i + 1], e[i + 2], e[i + 3]);
            }
            if constexpr (VEC == 8) {
                if (sr.out_f16) {  // the f32 value, rounded once to fp16
                    const size_t oi16 = (((size_t)b * a.G + g) * a.out_f16_blocks + a.blk_off + j) * a.D + d0;
                    st16_f16_checked(static_cast<__half*>(sr.out_f16) + oi16, e, f16_ovf);
                }
            }
        }
    } else if (a.state && active) {
        float* st = a.state + (((size_t)b * a.S + sr.state_series) * 3) * GD + (size_t)cv * VEC;
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
            st[i] = mx[i];
            st[GD + i] = l[i];
            st[2 * GD + i] = acc[i];
        }
    }
    if (f16_ovf) set_status(a.status, LBCA_ERR_UNSUPPORTED);
}

inline int round32(int n) { return (n + 31) / 32 * 32; }

template <typename T>
__global__ void __launch_bounds__(1024) ring_fill_kernel(const RingFillArgs a) {
    constexpr int VEC = Vec<T>::N;
    extern __shared__ __align__(16) float smem[];
    const int GD = a.G * a.D, NV = GD / VEC, NVH = a.D / VEC;
    const int b = blockIdx.y, tid = threadIdx.x;
    if (blockIdx.x == 0 && tid == 0) a.seq_lens[b] = a.T;
    if ((int)blockIdx.x >= a.n) return;  // uniform per CTA
    const int s = a.T - a.n + blockIdx.x;
    const bool active = tid < NV;
    const int cv = active ? tid : 0;
    float2* cs = reinterpret_cast<float2*>(smem);
    float* part = smem + a.rho;
    for (int k = tid; k < a.rho / 2; k += blockDim.x) cs[k] = rope_cs((int64_t)s, k, a.rope_step);
    __syncthreads();
    const int g = cv / NVH, d0 = (cv % NVH) * VEC;
    const size_t src = ((size_t)b * a.T + s) * GD + (size_t)cv * VEC;
    const size_t dst = (((size_t)b * a.G + g) * a.R + (s % a.R)) * a.D + d0;
    float e[VEC];
    if (active) ld16(static_cast<const T*>(a.k) + src, e);
    else
#pragma unroll
        for (int i = 0; i < VEC; ++i) e[i] = 0.f;
    // GQA form: the finalised key.  Shared form (no value series): the raw
    // entry as given, finalised by the decode kernels when they read it.
    if (a.v) {
        float ss = 0.f;
        if (a.rmsnorm) {
            float v = 0.f;
#pragma unroll
            for (int i = 0; i < VEC; ++i) v += e[i] * e[i];
            ss = head_sum(part, v, active ? tid - (cv % NVH) : 0, NVH);
        }
        finalise_key<T, VEC>(e, d0, a.D, a.rmsnorm, ss, a.eps, static_cast<const T*>(a.gamma), a.rho, cs);
    }
    if (active) {
        st16(static_cast<T*>(a.ring_k) + dst, e);
        if (a.v) {
            float vv[VEC];
            ld16(static_cast<const T*>(a.v) + src, vv);
            st16(static_cast<T*>(a.ring_v) + dst, vv);
        }
    }
}

// One CTA per sequence; threads [0, NV) carry the key series (or the shared
// entry), threads [NV, 2 NV) the value series.
template <typename T>
__global__ void __launch_bounds__(1024) append_kernel(const AppendArgs a) {
    constexpr int VEC = Vec<T>::N;
    extern __shared__ __align__(16) float smem[];
    const int GD = a.G * a.D, NV = GD / VEC, NVH = a.D / VEC;
    const int b = blockIdx.x, tid = threadIdx.x;
    const bool active = tid < a.S * NV;
    const int series = active ? tid / NV : 0;
    const int cv = active ? tid % NV : 0;
    const bool key = series == 0;
    const int pos = a.seq_lens[b];
    const int i = pos % a.m, j = pos / a.m;
    const bool complete = i == a.m - 1;

    float2* cs_raw = reinterpret_cast<float2*>(smem);
    float2* cs_pool = cs_raw + a.rho / 2;
    float* part = smem + 2 * a.rho;
    for (int k = tid; k < a.rho / 2; k += blockDim.x) {
        cs_raw[k] = rope_cs((int64_t)pos, k, a.rope_step);
        if (complete) cs_pool[k] = rope_cs((int64_t)j * a.m, k, a.rope_step);
    }
    __syncthreads();

    const int g = cv / NVH, d0 = (cv % NVH) * VEC;
    const size_t in = (size_t)b * GD + (size_t)cv * VEC;
    float x[VEC], z[VEC], bpv[VEC];
    if (active) {
        ld16(static_cast<const T*>(key ? a.k : a.v) + in, x);
        ld16(static_cast<const T*>(key ? a.zk : a.zv) + in, z);
        ld16(static_cast<const T*>(key ? a.bpk : a.bpv) + (size_t)i * GD + (size_t)cv * VEC, bpv);
    } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) { x[e] = 0.f; z[e] = 0.f; bpv[e] = 0.f; }
    }

    // running softmax of the open block (log2-domain max, sum, weighted sum)
    float* st = a.state + (((size_t)b * a.S + series) * 3) * GD + (size_t)cv * VEC;
    float mx[VEC], l[VEC], acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        const float av = (z[e] + bpv[e]) * kLog2e;
        if (i == 0 || !active) {
            mx[e] = av; l[e] = 1.f; acc[e] = x[e];
        } else {
            const float m0 = st[e], l0 = st[GD + e], a0 = st[2 * GD + e];
            const float mn = fmaxf(m0, av);
            const float r = ex2(m0 - mn), p = ex2(av - mn);
            mx[e] = mn;
            l[e] = l0 * r + p;
            acc[e] = fmaf(p, x[e], a0 * r);
        }
    }

    if (complete) {
        float e[VEC];
#pragma unroll
        for (int k = 0; k < VEC; ++k) e[k] = acc[k] / l[k];
        float ss = 0.f;
        if (a.rmsnorm) {
            float v = 0.f;
            if (key)
#pragma unroll
                for (int k = 0; k < VEC; ++k) v += e[k] * e[k];
            ss = head_sum(part, v, active ? tid - (cv % NVH) : 0, NVH);
        }
        if (key)
            finalise_key<T, VEC>(e, d0, a.D, a.rmsnorm, ss, a.eps, static_cast<const T*>(a.gamma),
                                 a.rho, cs_pool);
        if (active) {
            if (j < a.max_blocks) {
                T* o = static_cast<T*>(key ? a.pooled_k : a.pooled_v) +
                       (((size_t)b * a.G + g) * a.max_blocks + j) * a.D + d0;
                st16(o, e);
            } else {
                set_status(a.status, LBCA_ERR_CAPACITY);
            }
        }
    } else if (active) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            st[e] = mx[e];
            st[GD + e] = l[e];
            st[2 * GD + e] = acc[e];
        }
    }

    // the raw token joins the window: the finalised key (GQA form), the value
    // as is, or -- in the shared form, where the row is also the value -- the
    // raw entry as given, finalised in f32 by the decode kernels when read
    float r[VEC];
#pragma unroll
    for (int k = 0; k < VEC; ++k) r[k] = x[k];
    if (a.S == 2) {  // uniform across the CTA
        float ss = 0.f;
        if (a.rmsnorm) {
            float v = 0.f;
            if (key)
#pragma unroll
                for (int k = 0; k < VEC; ++k) v += r[k] * r[k];
            ss = head_sum(part, v, active ? tid - (cv % NVH) : 0, NVH);
        }
        if (key)
            finalise_key<T, VEC>(r, d0, a.D, a.rmsnorm, ss, a.eps, static_cast<const T*>(a.gamma), a.rho,
                                 cs_raw);
    }
    if (active) {
        T* o = static_cast<T*>(key ? a.ring_k : a.ring_v) +
               (((size_t)b * a.G + g) * a.R + (pos % a.R)) * a.D + d0;
        st16(o, r);
    }
    __syncthreads();
    if (tid == 0) a.seq_lens[b] = pos + 1;
}


}  // namespace

cudaError_t launch_pool(const PoolArgs& in, cudaStream_t s) {
    PoolArgs a = in;
    const int vec = a.dtype == LBCA_BF16 ? 8 : 4;
    const int nvh = a.D / vec;                 // <= 128 threads per head
    const int hpc = std::min(a.G, 256 / nvh);  // whole heads per CTA
    a.nblk = a.T / a.m + ((!a.dual && a.state && (a.T % a.m)) ? 1 : 0);
    if (a.nblk == 0 || a.B == 0 || a.nser < 1) return cudaSuccess;
    const int threads = round32(hpc * nvh);
    const size_t smem = (size_t)a.rho * 4 + (size_t)threads * 4;
    a.gz = (a.G + hpc - 1) / hpc;
    if (a.B > 65535 || (long long)a.gz * a.nser > 65535) return cudaErrorInvalidValue;
    dim3 grid(a.nblk, a.B, a.gz * a.nser);
    const bool raw = a.ser[0].raw_f16 || (a.nser > 1 && a.ser[1].raw_f16);
    if (a.dual && raw) return cudaErrorInvalidValue;
    if (a.dtype == LBCA_BF16) {
        if (a.dual)
            pool_kernel<__nv_bfloat16, false, true><<<grid, threads, smem, s>>>(a);
        else if (raw)
            pool_kernel<__nv_bfloat16, true, false><<<grid, threads, smem, s>>>(a);
        else
            pool_kernel<__nv_bfloat16, false, false><<<grid, threads, smem, s>>>(a);
    } else if (a.dual) {
        pool_kernel<float, false, true><<<grid, threads, smem, s>>>(a);
    } else {
        pool_kernel<float, false, false><<<grid, threads, smem, s>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_ring_fill(const RingFillArgs& a, cudaStream_t s) {
    if (a.B == 0) return cudaSuccess;
    const int vec = a.dtype == LBCA_BF16 ? 8 : 4;
    const int threads = round32(a.G * a.D / vec);
    const size_t smem = (size_t)a.rho * 4 + (size_t)threads * 4;
    dim3 grid(a.n > 0 ? a.n : 1, a.B);
    if (a.dtype == LBCA_BF16)
        ring_fill_kernel<__nv_bfloat16><<<grid, threads, smem, s>>>(a);
    else
        ring_fill_kernel<float><<<grid, threads, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t s) {
    if (a.B == 0) return cudaSuccess;
    const int vec = a.dtype == LBCA_BF16 ? 8 : 4;
    const int threads = round32(a.S * a.G * a.D / vec);
    const size_t smem = (size_t)a.rho * 8 + (size_t)threads * 4;
    if (a.dtype == LBCA_BF16)
        append_kernel<__nv_bfloat16><<<a.B, threads, smem, s>>>(a);
    else
        append_kernel<float><<<a.B, threads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace lbca
