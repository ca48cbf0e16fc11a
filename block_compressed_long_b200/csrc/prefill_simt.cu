// prefill_simt.cu -- causal block-compressed attention on CUDA cores (f32 math).
//
// Every query t attends, in one softmax, to the pooled entries j < P(t+1) and
// the raw tokens s in [P(t+1) m, t], plus the optional sink (mSeek README,
// "How LBCA works", steps 4-5; CSA page, "What is implemented").  Raw keys are
// finalised in the tile loader (RMSNorm, RoPE at s); pooled entries arrive
// finalised from the pooling kernel.
//
// This path serves the f32 I/O dtype (no TF32: every product is an f32 FMA)
// and the shapes the tensor-core kernel does not cover.  TPQ = max(4, D/32)
// lanes share a query (D/TPQ dims each, interleaved so that they read one
// contiguous 16*TPQ-byte span of a key row and the queries of a warp broadcast
// it); a CTA of 128 threads owns 128/TPQ queries of one head.  Key/value tiles
// (32 rows, 16 for D >= 256) are widened to f32 in shared memory; scores are
// taken eight keys at a time with one rescale.
#include "common.cuh"
#include "kernels.h"

namespace lbca {
namespace {

constexpr int NT = 128;

template <int D> struct Shape {
    static constexpr int TPQ = D / 32 > 4 ? D / 32 : 4;  // lanes per query
    static constexpr int QT = NT / TPQ;                   // queries per CTA
    static constexpr int KT = D >= 256 ? 16 : 32;         // key rows per tile
    static constexpr size_t smem = 2 * (size_t)KT * D * 4;
};

template <typename T, int D>
__global__ void __launch_bounds__(NT) prefill_simt_kernel(const PrefillArgs a) {
    constexpr int TPQ = Shape<D>::TPQ, QT = Shape<D>::QT, KT = Shape<D>::KT;
    constexpr int NC = D / (4 * TPQ);  // float4 chunks per thread
    extern __shared__ __align__(16) float smem[];
    float (*Ks)[D] = reinterpret_cast<float (*)[D]>(smem);
    float (*Vs)[D] = reinterpret_cast<float (*)[D]>(smem + KT * D);

    const int qt0 = blockIdx.x * QT, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int qi = tid / TPQ, j4 = tid % TPQ;
    const int g = h / (a.Hq / a.G);
    // query rows are local (0 .. T-1) at absolute positions t_off + row; raw
    // rows of k / v are local (0 .. T_raw-1) at absolute positions s_off + row
    const int tl = qt0 + qi;
    const bool qvalid = tl < a.T;
    const int t = a.t_off + tl;
    const int t_last = a.t_off + min(qt0 + QT, a.T) - 1;
    const int GD = a.G * a.D;

    // ---- query: load own dims, RMSNorm across the 4 lanes, RoPE at t ----
    float q[NC][4], o[NC][4];
    const T* qrow = static_cast<const T*>(a.q) + (((size_t)b * a.T + (qvalid ? tl : 0)) * a.Hq + h) * D;
#pragma unroll
    for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            q[c][i] = to_f<T>(qrow[4 * (j4 + TPQ * c) + i]);
            o[c][i] = 0.f;
        }
    if (a.rmsnorm) {
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c)
#pragma unroll
            for (int i = 0; i < 4; ++i) ss += q[c][i] * q[c][i];
#pragma unroll
        for (int off = 1; off < TPQ; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
        const T* gm = static_cast<const T*>(a.gamma_q);
#pragma unroll
        for (int c = 0; c < NC; ++c)
#pragma unroll
            for (int i = 0; i < 4; ++i) q[c][i] *= inv * (gm ? to_f<T>(gm[4 * (j4 + TPQ * c) + i]) : 1.f);
    }
    float2 qcs[NC][2];  // cos/sin at t for this thread's pairs (reused for the output rotation)
#pragma unroll
    for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
            const int d = 4 * (j4 + TPQ * c) + 2 * pr;
            qcs[c][pr] = make_float2(1.f, 0.f);
            if (a.rho && d >= D - a.rho) {
                qcs[c][pr] = rope_cs((int64_t)t, (d - (D - a.rho)) >> 1, a.rope_step);
                rotate_pair(q[c][2 * pr], q[c][2 * pr + 1], qcs[c][pr]);
            }
        }
    const float qscale = a.scale * kLog2e;
#pragma unroll
    for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) q[c][i] *= qscale;

    const int Pq = visible_blocks(t + 1, a.m, a.w);
    const int raw_lo = Pq * a.m;
    const int Pmax = visible_blocks(t_last + 1, a.m, a.w);
    const int s_lo = visible_blocks(a.t_off + qt0 + 1, a.m, a.w) * a.m;
    float mx = kNegInf, ls = 0.f;

    const size_t pool_head = ((size_t)b * a.G + g) * a.pool_stride;
    const int n_pool_tiles = (Pmax + KT - 1) / KT;
    const int n_raw_tiles = (t_last - s_lo + 1 + KT - 1) / KT;
    for (int tile = 0; tile < n_pool_tiles + n_raw_tiles; ++tile) {
        const bool pooled = tile < n_pool_tiles;
        const int base = pooled ? tile * KT : s_lo + (tile - n_pool_tiles) * KT;
        const int lim = pooled ? Pmax : t_last + 1;
        __syncthreads();
        // ---- load a tile: one warp per row, lanes over pairs of dims ----
        for (int rrow = warp; rrow < KT; rrow += NT / 32) {
            const int e = base + rrow;
            const bool ok = e < lim;
            if (pooled && a.pooled_f32) {
                const size_t o = (pool_head + (ok ? e : 0)) * D;
                const float* kr = static_cast<const float*>(a.pooled_k) + o;
                const float* vr = static_cast<const float*>(a.shared ? a.pooled_k : a.pooled_v) + o;
                for (int d = lane; d < D; d += 32) {
                    Ks[rrow][d] = ok ? kr[d] : 0.f;
                    Vs[rrow][d] = ok ? vr[d] : 0.f;
                }
            } else if (pooled) {
                const T* kr = static_cast<const T*>(a.pooled_k) + (pool_head + (ok ? e : 0)) * D;
                const T* vr = static_cast<const T*>(a.shared ? a.pooled_k : a.pooled_v) + (pool_head + (ok ? e : 0)) * D;
                for (int d = lane; d < D; d += 32) {
                    Ks[rrow][d] = ok ? to_f<T>(kr[d]) : 0.f;
                    Vs[rrow][d] = ok ? to_f<T>(vr[d]) : 0.f;
                }
            } else {
                const bool in_raw = ok && e >= a.s_off && e - a.s_off < a.T_raw;  // the host checks the span
                const size_t src = ((size_t)b * a.T_raw + (in_raw ? e - a.s_off : 0)) * GD + (size_t)g * D;
                const T* kr = static_cast<const T*>(a.k) + src;
                float ss = 0.f;
                for (int d = lane; d < D; d += 32) {
                    const float x = ok ? to_f<T>(kr[d]) : 0.f;
                    Ks[rrow][d] = x;
                    ss += x * x;
                }
                __syncwarp();
                if (a.rmsnorm) {
#pragma unroll
                    for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                    const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
                    const T* gm = static_cast<const T*>(a.gamma_kv);
                    for (int d = lane; d < D; d += 32) Ks[rrow][d] *= inv * (gm ? to_f<T>(gm[d]) : 1.f);
                    __syncwarp();
                }
                for (int d = 2 * lane; d < D; d += 64) {
                    if (a.rho && d >= D - a.rho && ok)
                        rotate_pair(Ks[rrow][d], Ks[rrow][d + 1],
                                    rope_cs((int64_t)e, (d - (D - a.rho)) >> 1, a.rope_step));
                }
                __syncwarp();
                if (a.shared) {
                    for (int d = lane; d < D; d += 32) Vs[rrow][d] = Ks[rrow][d];
                } else {
                    const T* vr = static_cast<const T*>(a.v) + src;
                    for (int d = lane; d < D; d += 32) Vs[rrow][d] = ok ? to_f<T>(vr[d]) : 0.f;
                }
            }
        }
        __syncthreads();
        // ---- scores and online softmax, 8 keys per step ----
        for (int e0 = 0; e0 < KT; e0 += 8) {
            float s[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                float acc = 0.f;
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    const float4 kv = *reinterpret_cast<const float4*>(&Ks[e0 + u][4 * (j4 + TPQ * c)]);
                    acc = fmaf(q[c][0], kv.x, acc);
                    acc = fmaf(q[c][1], kv.y, acc);
                    acc = fmaf(q[c][2], kv.z, acc);
                    acc = fmaf(q[c][3], kv.w, acc);
                }
#pragma unroll
                for (int off = 1; off < TPQ; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                const int e = base + e0 + u;
                const bool vis = qvalid && e < lim && (pooled ? e < Pq : (e >= raw_lo && e <= t));
                s[u] = vis ? acc : kNegInf;
            }
            float mn = mx;
#pragma unroll
            for (int u = 0; u < 8; ++u) mn = fmaxf(mn, s[u]);
            if (mn == kNegInf) continue;
            const float rr = ex2(mx - mn);
            float p[8];
            float psum = 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) { p[u] = ex2(s[u] - mn); psum += p[u]; }
            ls = fmaf(ls, rr, psum);
            mx = mn;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                float4 acc = make_float4(o[c][0] * rr, o[c][1] * rr, o[c][2] * rr, o[c][3] * rr);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float4 vv = *reinterpret_cast<const float4*>(&Vs[e0 + u][4 * (j4 + TPQ * c)]);
                    acc.x = fmaf(p[u], vv.x, acc.x);
                    acc.y = fmaf(p[u], vv.y, acc.y);
                    acc.z = fmaf(p[u], vv.z, acc.z);
                    acc.w = fmaf(p[u], vv.w, acc.w);
                }
                o[c][0] = acc.x; o[c][1] = acc.y; o[c][2] = acc.z; o[c][3] = acc.w;
            }
        }
    }

    if (!qvalid) return;
    float den = ls;
    if (a.sink) den += (mx == kNegInf) ? 1.0f : ex2(a.sink[h] * kLog2e - mx);
    const float inv = den > 0.f ? 1.0f / den : 0.f;
    T* orow = static_cast<T*>(a.out) + (((size_t)b * a.T + tl) * a.Hq + h) * D;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        float v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = o[c][i] * inv;
        if (a.shared && a.rho) {
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
                const int d = 4 * (j4 + TPQ * c) + 2 * pr;
                if (d >= D - a.rho)
                    rotate_pair(v[2 * pr], v[2 * pr + 1], make_float2(qcs[c][pr].x, -qcs[c][pr].y));
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) orow[4 * (j4 + TPQ * c) + i] = from_f<T>(v[i]);
    }
}

template <typename T, int D>
cudaError_t launch_d(const PrefillArgs& a, cudaStream_t s) {
    static bool attr_set[64] = {};  // per device
    const int dev_ = current_device();
    if (dev_ < 0 || !attr_set[dev_]) {
        cudaError_t e = cudaFuncSetAttribute(prefill_simt_kernel<T, D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Shape<D>::smem);
        if (e != cudaSuccess) return e;
        if (dev_ >= 0) attr_set[dev_] = true;
    }
    dim3 grid((a.T + Shape<D>::QT - 1) / Shape<D>::QT, a.Hq, a.B);
    prefill_simt_kernel<T, D><<<grid, NT, Shape<D>::smem, s>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch(const PrefillArgs& a, cudaStream_t s) {
    switch (a.D) {
        case 16: return launch_d<T, 16>(a, s);
        case 32: return launch_d<T, 32>(a, s);
        case 64: return launch_d<T, 64>(a, s);
        case 128: return launch_d<T, 128>(a, s);
        case 256: return launch_d<T, 256>(a, s);
        case 512: return launch_d<T, 512>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool prefill_simt_supported(int D) {
    return D == 16 || D == 32 || D == 64 || D == 128 || D == 256 || D == 512;
}

cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    if (a.dtype == LBCA_BF16) return dispatch<__nv_bfloat16>(a, s);
    return dispatch<float>(a, s);
}

}  // namespace lbca
