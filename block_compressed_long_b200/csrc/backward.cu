// backward.cu -- gradients of the prefill (block pooling + block-compressed
// attention) for training: the LBCA layers are trained by continued
// pretraining (mSeek README, "Experiment at a glance"), so the gradient of a
// loss reaches the queries, the raw keys and values, the pooling logits Z, the
// positional biases B_pos and the sink logits.
//
// Reverse-mode of the forward as defined (mSeek README, "How LBCA works",
// steps 2-5; HCA page, "What is implemented"; CSA page, "What is implemented"):
//   o_t = sum_e p_e val_e,  p = softmax over the visible entries and the sink
//   dS_e = p_e (dout_t . val_e - dout_t . o_t),  dq~_t = scale sum_e dS_e key_e,
//   dkey_e = scale sum_t dS_e q~_t,  dval_e = sum_t p_e dout_t,
//   d sink = -sum_t p_sink (dout_t . o_t),
// then back through RoPE (a rotation: its transpose turns by -pos), RMSNorm
// (dx = r g dy - x r^3 (g dy . x) / D) and the pooling softmax
// (dx_i = w_i dP, dz_i = db_i = w_i (x_i - P) dP).
//
// B200 mapping (CUDA cores, f32 arithmetic and gradients, f32 scratch):
//   1. pool_fwd    re-pools every complete block in f32 (one thread per
//                  channel; the backward needs the unrounded pooled values)
//   2. finalise    one warp per row: pooled keys, raw keys and queries
//                  finalised in f32; the output gradient turned by +t in the
//                  shared form; the row constant dout . out
//   3. row_lse     one warp per (row, head): log-sum-exp over the visible
//                  entries and the sink
//   4. dq          one warp per (row, head): dq~, then back through the
//                  query's RoPE and RMSNorm; sink gradient
//   5. dkv         one warp per (entry, kv head): the contiguous range of
//                  query rows that can see the entry, times the group's
//                  heads -- no atomics on key or value gradients
//   6. key_bwd     one warp per key row: back through RoPE and RMSNorm
//   7. pool_bwd    one thread per (block, channel): the pooling softmax's
//                  gradient into the raw inputs, the logits and (atomically
//                  over blocks) the bias
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace lbca {
namespace {

constexpr int kWarpsPerCta = 4;

template <typename T>
__device__ __forceinline__ float ldf(const T* p) { return to_f<T>(*p); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Row helpers: lane holds dims lane, lane + 32, ... (NPL = D / 32 of them).
template <int NPL>
__device__ __forceinline__ float row_dot(const float (&a)[NPL], const float* b, int lane) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) s = fmaf(a[i], b[lane + 32 * i], s);
    return warp_sum(s);
}

// RoPE of the row held by the warp at position pos (sign -1: the inverse turn).
// Pairs (2k, 2k+1) of the last rho dims; the partner dim lives in lane ^ 1.
template <int NPL>
__device__ __forceinline__ void row_rope(float (&x)[NPL], int lane, int D, int rho, double step, int64_t pos) {
    if (!rho) return;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int d = lane + 32 * i;
        const float other = __shfl_xor_sync(0xffffffffu, x[i], 1);
        if (d >= D - rho) {
            const float2 cs = rope_cs(pos, (d - (D - rho)) >> 1, step);
            x[i] = (d & 1) == 0 ? x[i] * cs.x - other * cs.y : other * cs.y + x[i] * cs.x;
        }
    }
}

// RMSNorm of a row (gamma [D] of type T or null).
template <int NPL, typename T>
__device__ __forceinline__ void row_rms(float (&x)[NPL], int lane, int D, float eps, const T* gamma) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) ss = fmaf(x[i], x[i], ss);
    const float r = 1.0f / sqrtf(warp_sum(ss) / (float)D + eps);
#pragma unroll
    for (int i = 0; i < NPL; ++i) x[i] *= r * (gamma ? ldf(gamma + lane + 32 * i) : 1.f);
}

// dx of RMSNorm given the input row x and dy.
template <int NPL, typename T>
__device__ __forceinline__ void row_rms_bwd(const float (&x)[NPL], float (&dy)[NPL], int lane, int D, float eps,
                                            const T* gamma) {
    float ss = 0.f, dot = 0.f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const float gm = gamma ? ldf(gamma + lane + 32 * i) : 1.f;
        ss = fmaf(x[i], x[i], ss);
        dot = fmaf(gm * dy[i], x[i], dot);
    }
    ss = warp_sum(ss);
    dot = warp_sum(dot);
    const float r = 1.0f / sqrtf(ss / (float)D + eps);
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const float gm = gamma ? ldf(gamma + lane + 32 * i) : 1.f;
        dy[i] = r * gm * dy[i] - x[i] * r * r * r * dot / (float)D;
    }
}

// Visible list of query row t: P pooled entries, then raw tokens [s0, t].
struct Vis {
    int P, s0, n;
};
__device__ __forceinline__ Vis vis_of(const BwdArgs& a, int t) {
    Vis v;
    v.P = visible_blocks(t + 1, a.m, a.w);
    v.s0 = v.P * a.m;
    v.n = v.P + (t - v.s0 + 1);
    return v;
}

// f32 row of visible entry e of (b, g) for row t's list: key and value.
__device__ __forceinline__ const float* key_row(const BwdArgs& a, int b, int g, const Vis& v, int e) {
    return e < v.P ? a.Ef + (((size_t)b * a.NB + e) * a.G + g) * a.D
                   : a.Kf + (((size_t)b * a.T + v.s0 + (e - v.P)) * a.G + g) * a.D;
}

// ---- 1. f32 re-pooling of every complete block (value: pooled; key: before finalisation) ----
template <typename T>
__global__ void pool_fwd_kernel(const BwdArgs a) {
    const int GD = a.G * a.D;
    const size_t n = (size_t)a.S * a.B * a.NB * GD;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < n; idx += (size_t)gridDim.x * blockDim.x) {
        const int col = (int)(idx % GD);
        const size_t j = (idx / GD) % a.NB;
        const size_t b = (idx / ((size_t)GD * a.NB)) % a.B;
        const int sr = (int)(idx / ((size_t)GD * a.NB * a.B));
        const T* x = static_cast<const T*>(sr ? a.v : a.k) + (b * a.T + j * a.m) * GD + col;
        const T* z = static_cast<const T*>(sr ? a.zv : a.zk) + (b * a.T + j * a.m) * GD + col;
        const T* bp = static_cast<const T*>(sr ? a.bpv : a.bpk) + col;
        float mx = kNegInf;
        for (int i = 0; i < a.m; ++i) mx = fmaxf(mx, ldf(z + (size_t)i * GD) + ldf(bp + (size_t)i * GD));
        float den = 0.f, num = 0.f;
        for (int i = 0; i < a.m; ++i) {
            const float p = expf(ldf(z + (size_t)i * GD) + ldf(bp + (size_t)i * GD) - mx);
            den += p;
            num = fmaf(p, ldf(x + (size_t)i * GD), num);
        }
        const float P = num / den;
        if (sr == 0) a.Pk[idx] = P;
        a.Ef[idx] = P;  // keys finalised in place by the next kernel
    }
}

// ---- 2. finalised pooled keys, raw keys, queries; turned dout; dout . out ----
template <typename T, int NPL>
__global__ void finalise_kernel(const BwdArgs a) {
    const int lane = threadIdx.x & 31;
    const size_t w = blockIdx.x * (size_t)kWarpsPerCta + (threadIdx.x >> 5);
    const size_t nk = (size_t)a.B * a.NB * a.G, nr = (size_t)a.B * a.T * a.G, nq = (size_t)a.B * a.T * a.Hq;
    const int D = a.D;
    float x[NPL];
    if (w < nk) {  // pooled key (b, j, g), in place
        float* row = a.Ef + w * D;
        const int j = (int)((w / a.G) % a.NB);
#pragma unroll
        for (int i = 0; i < NPL; ++i) x[i] = row[lane + 32 * i];
        if (a.rmsnorm) row_rms<NPL>(x, lane, D, a.eps, static_cast<const T*>(a.gamma_kv));
        row_rope<NPL>(x, lane, D, a.rho, a.rope_step, (int64_t)j * a.m);
#pragma unroll
        for (int i = 0; i < NPL; ++i) row[lane + 32 * i] = x[i];
    } else if (w < nk + nr) {  // raw key (b, s, g)
        const size_t r = w - nk;
        const int s = (int)((r / a.G) % a.T);
        const T* src = static_cast<const T*>(a.k) + r * D;
#pragma unroll
        for (int i = 0; i < NPL; ++i) x[i] = ldf(src + lane + 32 * i);
        if (a.rmsnorm) row_rms<NPL>(x, lane, D, a.eps, static_cast<const T*>(a.gamma_kv));
        row_rope<NPL>(x, lane, D, a.rho, a.rope_step, s);
#pragma unroll
        for (int i = 0; i < NPL; ++i) a.Kf[r * D + lane + 32 * i] = x[i];
        if (!a.shared) {  // the raw value, widened (GQA)
            const T* vs = static_cast<const T*>(a.v) + r * D;
#pragma unroll
            for (int i = 0; i < NPL; ++i) a.vf[r * D + lane + 32 * i] = ldf(vs + lane + 32 * i);
        }
    } else if (w < nk + nr + nq) {  // query (b, t, h): finalised; dout turned; dout . out
        const size_t r = w - nk - nr;
        const int t = (int)((r / a.Hq) % a.T);
        const T* src = static_cast<const T*>(a.q) + r * D;
#pragma unroll
        for (int i = 0; i < NPL; ++i) x[i] = ldf(src + lane + 32 * i);
        if (a.rmsnorm) row_rms<NPL>(x, lane, D, a.eps, static_cast<const T*>(a.gamma_q));
        row_rope<NPL>(x, lane, D, a.rho, a.rope_step, t);
#pragma unroll
        for (int i = 0; i < NPL; ++i) a.qf[r * D + lane + 32 * i] = x[i];
        float dy[NPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) dy[i] = ldf(static_cast<const T*>(a.dout) + r * D + lane + 32 * i);
        if (a.shared) row_rope<NPL>(dy, lane, D, a.rho, a.rope_step, t);  // d o = R(t) d out
#pragma unroll
        for (int i = 0; i < NPL; ++i) a.dof[r * D + lane + 32 * i] = dy[i];
    }
}

// Value row of visible entry e (the key row in the shared form).
__device__ __forceinline__ const float* val_row(const BwdArgs& a, int b, int g, const Vis& v, int e) {
    if (a.shared) return key_row(a, b, g, v, e);
    return e < v.P ? a.Ef + ((((size_t)a.B + b) * a.NB + e) * a.G + g) * a.D
                   : a.vf + (((size_t)b * a.T + v.s0 + (e - v.P)) * a.G + g) * a.D;
}

// ---- 3. per (row, head): log-sum-exp over the visible entries and the sink, and
// the row constant d o . o with the output recomputed in f32 ----
template <int NPL>
__global__ void row_lse_kernel(const BwdArgs a) {
    const int lane = threadIdx.x & 31;
    const size_t r = blockIdx.x * (size_t)kWarpsPerCta + (threadIdx.x >> 5);  // (b, t, h)
    if (r >= (size_t)a.B * a.T * a.Hq) return;
    const int h = (int)(r % a.Hq), t = (int)((r / a.Hq) % a.T), b = (int)(r / ((size_t)a.Hq * a.T));
    const int g = h / (a.Hq / a.G);
    float q[NPL], o[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        q[i] = a.qf[r * a.D + lane + 32 * i] * a.scale;
        o[i] = 0.f;
    }
    const Vis v = vis_of(a, t);
    float M = a.sink ? a.sink[h] : kNegInf, l = a.sink ? 1.f : 0.f;
    for (int e = 0; e < v.n; ++e) {
        const float s = row_dot<NPL>(q, key_row(a, b, g, v, e), lane);
        const float* vr = val_row(a, b, g, v, e);
        float c = 1.f, p = 1.f;  // rescale of what is there, weight of the new entry
        if (s > M) {
            c = expf(M - s);
            M = s;
        } else {
            p = expf(s - M);
        }
        l = l * c + p;
#pragma unroll
        for (int i = 0; i < NPL; ++i) o[i] = fmaf(p, vr[lane + 32 * i], o[i] * c);
    }
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) dot = fmaf(a.dof[r * a.D + lane + 32 * i], o[i], dot);
    dot = warp_sum(dot);
    if (lane == 0) {
        a.lse[r] = M + logf(l);
        a.dsum[r] = dot / l;
    }
}

// ---- 4. dq: back through the scores, the query's RoPE and RMSNorm; sink gradient ----
template <typename T, int NPL>
__global__ void dq_kernel(const BwdArgs a) {
    const int lane = threadIdx.x & 31;
    const size_t r = blockIdx.x * (size_t)kWarpsPerCta + (threadIdx.x >> 5);
    if (r >= (size_t)a.B * a.T * a.Hq) return;
    const int h = (int)(r % a.Hq), t = (int)((r / a.Hq) % a.T), b = (int)(r / ((size_t)a.Hq * a.T));
    const int g = h / (a.Hq / a.G);
    float q[NPL], dof[NPL], acc[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        q[i] = a.qf[r * a.D + lane + 32 * i] * a.scale;
        dof[i] = a.dof[r * a.D + lane + 32 * i];
        acc[i] = 0.f;
    }
    const float lse = a.lse[r], dsum = a.dsum[r];
    const Vis v = vis_of(a, t);
    for (int e = 0; e < v.n; ++e) {
        const float* kr = key_row(a, b, g, v, e);
        const float* vr = val_row(a, b, g, v, e);
        const float p = expf(row_dot<NPL>(q, kr, lane) - lse);
        const float dS = p * (row_dot<NPL>(dof, vr, lane) - dsum);
#pragma unroll
        for (int i = 0; i < NPL; ++i) acc[i] = fmaf(dS * a.scale, kr[lane + 32 * i], acc[i]);
    }
    if (a.sink && lane == 0) atomicAdd(a.dsink + h, -expf(a.sink[h] - lse) * dsum);
    // back through RoPE at t (the inverse turn) and RMSNorm
    row_rope<NPL>(acc, lane, a.D, a.rho, a.rope_step, -(int64_t)t);
    if (a.rmsnorm) {
        float x[NPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) x[i] = ldf(static_cast<const T*>(a.q) + r * a.D + lane + 32 * i);
        row_rms_bwd<NPL>(x, acc, lane, a.D, a.eps, static_cast<const T*>(a.gamma_q));
    }
#pragma unroll
    for (int i = 0; i < NPL; ++i) a.dq[r * a.D + lane + 32 * i] = acc[i];
}

// ---- 5. dkey, dval of each entry over the rows that can see it ----
// Pooled block j is visible to rows t >= (j+1) m + w - 1; raw token s to rows
// t in [s, (floor(s/m)+1) m + w - 2] (block-aligned partition).
template <int NPL>
__global__ void dkv_kernel(const BwdArgs a) {
    const int lane = threadIdx.x & 31;
    const size_t wi = blockIdx.x * (size_t)kWarpsPerCta + (threadIdx.x >> 5);
    const size_t npool = (size_t)a.B * a.NB * a.G, nraw = (size_t)a.B * a.T * a.G;
    if (wi >= npool + nraw) return;
    const bool pooled = wi < npool;
    const size_t r = pooled ? wi : wi - npool;
    const int g = (int)(r % a.G);
    const int pos = (int)((r / a.G) % (pooled ? a.NB : a.T));  // block j or token s
    const int b = (int)(r / ((size_t)a.G * (pooled ? a.NB : a.T)));
    const int rg = a.Hq / a.G;
    int t_lo, t_hi;
    if (pooled) {
        t_lo = (pos + 1) * a.m + a.w - 1;
        t_hi = a.T - 1;
    } else {
        t_lo = pos;
        t_hi = min(a.T - 1, (pos / a.m + 1) * a.m + a.w - 2);
    }
    const float* kr = pooled ? a.Ef + r * a.D : a.Kf + r * a.D;
    const float* vr = a.shared ? kr : (pooled ? a.Ef + (npool + r) * a.D : a.vf + r * a.D);
    float key[NPL], val[NPL], dk[NPL], dv[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        key[i] = kr[lane + 32 * i];
        val[i] = vr[lane + 32 * i];
        dk[i] = 0.f;
        dv[i] = 0.f;
    }
    for (int t = t_lo; t <= t_hi; ++t) {
        for (int hh = 0; hh < rg; ++hh) {
            const size_t row = ((size_t)b * a.T + t) * a.Hq + (size_t)g * rg + hh;
            const float* qr = a.qf + row * a.D;
            const float* dr = a.dof + row * a.D;
            const float p = expf(row_dot<NPL>(key, qr, lane) * a.scale - a.lse[row]);
            const float dS = p * (row_dot<NPL>(val, dr, lane) - a.dsum[row]);
#pragma unroll
            for (int i = 0; i < NPL; ++i) {
                dk[i] = fmaf(dS * a.scale, qr[lane + 32 * i], dk[i]);
                dv[i] = fmaf(p, dr[lane + 32 * i], dv[i]);
            }
        }
    }
    float* dko = pooled ? a.dE + r * a.D : a.dKf + r * a.D;
    float* dvo = a.shared ? dko : (pooled ? a.dE + (npool + r) * a.D : a.dv + r * a.D);
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const float x = a.shared ? dk[i] + dv[i] : dk[i];
        dko[lane + 32 * i] = x;
        if (!a.shared) dvo[lane + 32 * i] = dv[i];
    }
}

// ---- 6. back through the key finalisation (pooled and raw key rows) ----
template <typename T, int NPL>
__global__ void key_bwd_kernel(const BwdArgs a) {
    const int lane = threadIdx.x & 31;
    const size_t w = blockIdx.x * (size_t)kWarpsPerCta + (threadIdx.x >> 5);
    const size_t nk = (size_t)a.B * a.NB * a.G, nr = (size_t)a.B * a.T * a.G;
    if (w >= nk + nr) return;
    const bool pooled = w < nk;
    const size_t r = pooled ? w : w - nk;
    const int64_t pos = pooled ? (int64_t)((r / a.G) % a.NB) * a.m : (int64_t)((r / a.G) % a.T);
    float dy[NPL], x[NPL];
    const float* src = pooled ? a.dE + r * a.D : a.dKf + r * a.D;
#pragma unroll
    for (int i = 0; i < NPL; ++i) dy[i] = src[lane + 32 * i];
    row_rope<NPL>(dy, lane, a.D, a.rho, a.rope_step, -pos);
    if (a.rmsnorm) {
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            x[i] = pooled ? a.Pk[r * a.D + lane + 32 * i] : ldf(static_cast<const T*>(a.k) + r * a.D + lane + 32 * i);
        row_rms_bwd<NPL>(x, dy, lane, a.D, a.eps, static_cast<const T*>(a.gamma_kv));
    }
    float* dst = pooled ? a.dE + r * a.D : a.dk + r * a.D;
#pragma unroll
    for (int i = 0; i < NPL; ++i) dst[lane + 32 * i] = dy[i];
}

// ---- 7. the pooling softmax: raw inputs, logits and bias of every complete block ----
template <typename T>
__global__ void pool_bwd_kernel(const BwdArgs a) {
    const int GD = a.G * a.D;
    const size_t n = (size_t)a.S * a.B * a.NB * GD;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < n; idx += (size_t)gridDim.x * blockDim.x) {
        const int col = (int)(idx % GD);
        const size_t j = (idx / GD) % a.NB;
        const size_t b = (idx / ((size_t)GD * a.NB)) % a.B;
        const int sr = (int)(idx / ((size_t)GD * a.NB * a.B));
        const size_t tok0 = (b * a.T + j * a.m) * GD + col;
        const T* x = static_cast<const T*>(sr ? a.v : a.k) + tok0;
        const T* z = static_cast<const T*>(sr ? a.zv : a.zk) + tok0;
        const T* bp = static_cast<const T*>(sr ? a.bpv : a.bpk) + col;
        float* dx = (sr ? a.dv : a.dk) + tok0;
        float* dz = (sr ? a.dzv : a.dzk) + tok0;
        float* db = (sr ? a.dbv : a.dbk) + col;
        const float dP = a.dE[idx];           // d of the pooled value (keys: before finalisation)
        const float P = sr ? a.Ef[idx] : a.Pk[idx];
        float mx = kNegInf;
        for (int i = 0; i < a.m; ++i) mx = fmaxf(mx, ldf(z + (size_t)i * GD) + ldf(bp + (size_t)i * GD));
        float den = 0.f;
        for (int i = 0; i < a.m; ++i) den += expf(ldf(z + (size_t)i * GD) + ldf(bp + (size_t)i * GD) - mx);
        for (int i = 0; i < a.m; ++i) {
            const float wgt = expf(ldf(z + (size_t)i * GD) + ldf(bp + (size_t)i * GD) - mx) / den;
            const float da = wgt * (ldf(x + (size_t)i * GD) - P) * dP;
            dx[(size_t)i * GD] += wgt * dP;
            dz[(size_t)i * GD] = da;
            atomicAdd(db + (size_t)i * GD, da);
        }
    }
}

// ---- register-tiled passes over (row, entry) pairs, D = 64 or 128 ----
// The pairs a query row sees form, per tile of RT consecutive rows of one head,
// a prefix of the pooled entries and a band of raw tokens; per tile of ET
// entries of one kv head, a range of rows.  Tiles of both sides are staged in
// shared memory and every thread computes a small block of scores (and of the
// outputs) in registers, so each K/V and Q/dO row is read once per tile
// instead of once per pair.
constexpr int kTT = 256;   // threads of the tiled passes
constexpr int RT = 64;     // query rows per tile
constexpr int ET = 32;     // entries per tile

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ float dot4(float4 x, float4 y, float acc) {
    return fmaf(x.w, y.w, fmaf(x.z, y.z, fmaf(x.y, y.y, fmaf(x.x, y.x, acc))));
}
__device__ __forceinline__ void axpy4(float a, float4 x, float* y) {
    y[0] = fmaf(a, x.x, y[0]);
    y[1] = fmaf(a, x.y, y[1]);
    y[2] = fmaf(a, x.z, y[2]);
    y[3] = fmaf(a, x.w, y[3]);
}

// Entry `idx` (pooled block, or raw token) visible to row t, P = P(t + 1).
__device__ __forceinline__ bool sees(bool pooled, int idx, int t, int P, int m) {
    return pooled ? idx < P : (idx >= P * m && idx <= t);
}

// f32 key and value rows of entry idx of (b, g) into Ks, Vs (row r); zeros past cnt.
template <int D>
__device__ __forceinline__ void load_entries(const BwdArgs& a, bool pooled, int base, int cnt, int b, int g, float* Ks,
                                             float* Vs) {
    constexpr int LD = D + 4;
    for (int i = threadIdx.x; i < ET * (D / 4); i += kTT) {
        const int r = i / (D / 4), c = 4 * (i % (D / 4));
        float4 k4 = make_float4(0.f, 0.f, 0.f, 0.f), v4 = k4;
        if (r < cnt) {
            const int e = base + r;
            const size_t kr = pooled ? (((size_t)b * a.NB + e) * a.G + g) : (((size_t)b * a.T + e) * a.G + g);
            const float* kp = (pooled ? a.Ef : a.Kf) + kr * D;
            const float* vp = a.shared ? kp
                                       : (pooled ? a.Ef + ((size_t)a.B * a.NB * a.G + kr) * D : a.vf + kr * D);
            k4 = ld4(kp + c);
            v4 = ld4(vp + c);
        }
        st4(Ks + r * LD + c, k4);
        st4(Vs + r * LD + c, v4);
    }
}

template <int D>
constexpr size_t row_pass_smem() {
    return (size_t)(2 * RT * (D + 4) + 2 * ET * (D + 4) + RT * (ET + 1)) * 4 + RT * 4 + 64;
}

// ---- 3+4 (tiled). Per tile of RT rows of one head: sweep 1 -- log-sum-exp and
// the output (for dsum = dout . o); sweep 2 -- dS and dq~ = scale sum dS key.
// dq~ goes to dq; the turn back through RoPE and RMSNorm follows (dq_tail).
template <int D>
__global__ void __launch_bounds__(kTT, 2) row_pass_kernel(const BwdArgs a) {
    constexpr int LD = D + 4, NC = D / 32;
    extern __shared__ __align__(16) float sm[];
    float* Qs = sm;
    float* dOs = Qs + RT * LD;
    float* Ks = dOs + RT * LD;
    float* Vs = Ks + ET * LD;
    float* Ps = Vs + ET * LD;                        // [RT][ET + 1]
    int* Prow = reinterpret_cast<int*>(Ps + RT * (ET + 1));
    float* red = reinterpret_cast<float*>(Prow + RT);  // [kTT / 32]

    const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7, lane = tid & 31;
    // later row tiles see more pooled entries: they are launched first, so the
    // grid's last wave holds the short ones
    const int t0 = (gridDim.x - 1 - blockIdx.x) * RT, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (a.Hq / a.G);
    const int nrow = min(RT, a.T - t0);
    for (int i = tid; i < RT * (D / 4); i += kTT) {
        const int r = i / (D / 4), c = 4 * (i % (D / 4));
        float4 q4 = make_float4(0.f, 0.f, 0.f, 0.f), d4 = q4;
        if (r < nrow) {
            const size_t row = ((size_t)b * a.T + t0 + r) * a.Hq + h;
            q4 = ld4(a.qf + row * D + c);
            q4.x *= a.scale; q4.y *= a.scale; q4.z *= a.scale; q4.w *= a.scale;
            d4 = ld4(a.dof + row * D + c);
        }
        st4(Qs + r * LD + c, q4);
        st4(dOs + r * LD + c, d4);
    }
    for (int r = tid; r < RT; r += kTT) Prow[r] = visible_blocks(t0 + r + 1, a.m, a.w);
    const int t_last = t0 + nrow - 1;
    const int Pmax = visible_blocks(t_last + 1, a.m, a.w);
    const int s_lo = visible_blocks(t0 + 1, a.m, a.w) * a.m;
    const int npt = (Pmax + ET - 1) / ET, nrt = (t_last - s_lo + 1 + ET - 1) / ET;
    const int r0 = 2 * ty;
    const float sink = a.sink ? a.sink[h] : kNegInf;

    float M[2], l[2], o[2][4 * NC];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        M[i] = sink;
        l[i] = a.sink ? 1.f : 0.f;
#pragma unroll
        for (int c = 0; c < 4 * NC; ++c) o[i][c] = 0.f;
    }
    // ---- sweep 1 ----
    for (int tile = 0; tile < npt + nrt; ++tile) {
        const bool pooled = tile < npt;
        const int base = pooled ? tile * ET : s_lo + (tile - npt) * ET;
        const int cnt = min(ET, pooled ? Pmax - base : t_last + 1 - base);
        __syncthreads();  // the previous tile's K, V, P are consumed
        load_entries<D>(a, pooled, base, cnt, b, g, Ks, Vs);
        __syncthreads();
        float sc[2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[i][e] = 0.f;
#pragma unroll 4
        for (int d = 0; d < D; d += 4) {
            const float4 q0 = ld4(Qs + r0 * LD + d), q1 = ld4(Qs + (r0 + 1) * LD + d);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float4 k4 = ld4(Ks + (tx + 8 * e) * LD + d);
                sc[0][e] = dot4(q0, k4, sc[0][e]);
                sc[1][e] = dot4(q1, k4, sc[1][e]);
            }
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = r0 + i, t = t0 + r;
            float mx = kNegInf;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int ee = tx + 8 * e;
                const bool ok = r < nrow && ee < cnt && sees(pooled, base + ee, t, Prow[r], a.m);
                sc[i][e] = ok ? sc[i][e] : kNegInf;
                mx = fmaxf(mx, sc[i][e]);
            }
#pragma unroll
            for (int off = 1; off < 8; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float mn = fmaxf(M[i], mx);
            const float c = mn == kNegInf ? 1.f : expf(M[i] - mn);
            float ps = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float p = sc[i][e] == kNegInf ? 0.f : expf(sc[i][e] - mn);
                ps += p;
                Ps[r * (ET + 1) + tx + 8 * e] = p;
            }
#pragma unroll
            for (int off = 1; off < 8; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
            l[i] = l[i] * c + ps;
            M[i] = mn;
#pragma unroll
            for (int k = 0; k < 4 * NC; ++k) o[i][k] *= c;
        }
        __syncthreads();
        for (int e = 0; e < cnt; ++e) {
            const float p0 = Ps[r0 * (ET + 1) + e], p1 = Ps[(r0 + 1) * (ET + 1) + e];
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const float4 v4 = ld4(Vs + e * LD + 32 * c + 4 * tx);
                axpy4(p0, v4, &o[0][4 * c]);
                axpy4(p1, v4, &o[1][4 * c]);
            }
        }
    }
    // ---- log-sum-exp, dout . o / l; the sink's gradient ----
    float lse[2], dsum[2], sink_g = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = r0 + i;
        float dt = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const float4 d4 = ld4(dOs + r * LD + 32 * c + 4 * tx);
            dt = fmaf(d4.x, o[i][4 * c], fmaf(d4.y, o[i][4 * c + 1], fmaf(d4.z, o[i][4 * c + 2], fmaf(d4.w, o[i][4 * c + 3], dt))));
        }
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) dt += __shfl_xor_sync(0xffffffffu, dt, off);
        lse[i] = M[i] + logf(l[i]);
        dsum[i] = dt / l[i];
        if (r < nrow && tx == 0) {
            const size_t row = ((size_t)b * a.T + t0 + r) * a.Hq + h;
            a.lse[row] = lse[i];
            a.dsum[row] = dsum[i];
            if (a.sink) sink_g -= expf(sink - lse[i]) * dsum[i];
        }
    }
    // ---- sweep 2: dq~ ----
    float dq[2][4 * NC];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int c = 0; c < 4 * NC; ++c) dq[i][c] = 0.f;
    for (int tile = 0; tile < npt + nrt; ++tile) {
        const bool pooled = tile < npt;
        const int base = pooled ? tile * ET : s_lo + (tile - npt) * ET;
        const int cnt = min(ET, pooled ? Pmax - base : t_last + 1 - base);
        __syncthreads();
        load_entries<D>(a, pooled, base, cnt, b, g, Ks, Vs);
        __syncthreads();
        float sc[2][4], dp[2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[i][e] = dp[i][e] = 0.f;
#pragma unroll 2
        for (int d = 0; d < D; d += 4) {
            const float4 q0 = ld4(Qs + r0 * LD + d), q1 = ld4(Qs + (r0 + 1) * LD + d);
            const float4 g0 = ld4(dOs + r0 * LD + d), g1 = ld4(dOs + (r0 + 1) * LD + d);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float4 k4 = ld4(Ks + (tx + 8 * e) * LD + d);
                const float4 v4 = ld4(Vs + (tx + 8 * e) * LD + d);
                sc[0][e] = dot4(q0, k4, sc[0][e]);
                sc[1][e] = dot4(q1, k4, sc[1][e]);
                dp[0][e] = dot4(g0, v4, dp[0][e]);
                dp[1][e] = dot4(g1, v4, dp[1][e]);
            }
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = r0 + i, t = t0 + r;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int ee = tx + 8 * e;
                const bool ok = r < nrow && ee < cnt && sees(pooled, base + ee, t, Prow[r], a.m);
                Ps[r * (ET + 1) + ee] = ok ? expf(sc[i][e] - lse[i]) * (dp[i][e] - dsum[i]) * a.scale : 0.f;
            }
        }
        __syncthreads();
        for (int e = 0; e < cnt; ++e) {
            const float s0 = Ps[r0 * (ET + 1) + e], s1 = Ps[(r0 + 1) * (ET + 1) + e];
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const float4 k4 = ld4(Ks + e * LD + 32 * c + 4 * tx);
                axpy4(s0, k4, &dq[0][4 * c]);
                axpy4(s1, k4, &dq[1][4 * c]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = r0 + i;
        if (r >= nrow) continue;
        const size_t row = ((size_t)b * a.T + t0 + r) * a.Hq + h;
#pragma unroll
        for (int c = 0; c < NC; ++c)
            st4(a.dq + row * D + 32 * c + 4 * tx,
                make_float4(dq[i][4 * c], dq[i][4 * c + 1], dq[i][4 * c + 2], dq[i][4 * c + 3]));
    }
    if (a.sink) {  // one atomic per CTA
        float v = sink_g;
#pragma unroll
        for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) red[tid >> 5] = v;
        __syncthreads();
        if (tid == 0) {
            float s = 0.f;
            for (int w = 0; w < kTT / 32; ++w) s += red[w];
            atomicAdd(a.dsink + h, s);
        }
    }
}

// dq~ (in dq) back through the query's RoPE at t and RMSNorm, one warp per row.
template <typename T, int NPL>
__global__ void dq_tail_kernel(const BwdArgs a) {
    const int lane = threadIdx.x & 31;
    const size_t r = blockIdx.x * (size_t)kWarpsPerCta + (threadIdx.x >> 5);
    if (r >= (size_t)a.B * a.T * a.Hq) return;
    const int t = (int)((r / a.Hq) % a.T);
    float acc[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) acc[i] = a.dq[r * a.D + lane + 32 * i];
    row_rope<NPL>(acc, lane, a.D, a.rho, a.rope_step, -(int64_t)t);
    if (a.rmsnorm) {
        float x[NPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) x[i] = ldf(static_cast<const T*>(a.q) + r * a.D + lane + 32 * i);
        row_rms_bwd<NPL>(x, acc, lane, a.D, a.eps, static_cast<const T*>(a.gamma_q));
    }
#pragma unroll
    for (int i = 0; i < NPL; ++i) a.dq[r * a.D + lane + 32 * i] = acc[i];
}

template <int D>
constexpr size_t entry_pass_smem() {
    return (size_t)(2 * ET * (D + 4) + 2 * RT * (D + 4) + 2 * ET * (RT + 1)) * 4 + 3 * RT * 4;
}

// ---- 5 (tiled). Per tile of ET entries of one kv head: dkey and dval over the
// rows (of every head of the group) that can see the tile's entries.  A pooled
// tile is seen by every later row, so its rows are cut into chunks of kRowChunk
// row tiles, one CTA each, whose sums are added into the (zeroed) entry
// gradients; a raw tile's few rows stay with one CTA, which stores its sums.
constexpr int kRowChunk = 4;
template <int D>
__global__ void __launch_bounds__(kTT, 1) entry_pass_kernel(const BwdArgs a) {
    constexpr int LD = D + 4, NC = D / 64;
    extern __shared__ __align__(16) float sm[];
    float* Ks = sm;
    float* Vs = Ks + ET * LD;
    float* Qs = Vs + ET * LD;
    float* dOs = Qs + RT * LD;
    float* PT = dOs + RT * LD;              // [ET][RT + 1]
    float* dST = PT + ET * (RT + 1);         // [ET][RT + 1]
    float* lse_s = dST + ET * (RT + 1);
    float* dsum_s = lse_s + RT;
    int* Prow = reinterpret_cast<int*>(dsum_s + RT);

    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int g = blockIdx.y, b = blockIdx.z, rg = a.Hq / a.G;
    const int nchunk = (a.T + RT * kRowChunk - 1) / (RT * kRowChunk);
    const int npt = (a.NB + ET - 1) / ET * nchunk;
    const bool pooled = (int)blockIdx.x < npt;
    const int base = pooled ? (blockIdx.x / nchunk) * ET : (blockIdx.x - npt) * ET;
    const int cnt = min(ET, (pooled ? a.NB : a.T) - base);
    // rows that can see some entry of the tile (for a pooled tile, within this CTA's chunk)
    int t_lo, t_hi;
    if (pooled) {
        const int c0 = (blockIdx.x % nchunk) * RT * kRowChunk;
        t_lo = max((base + 1) * a.m + a.w - 1, c0);
        t_hi = min(a.T - 1, c0 + RT * kRowChunk - 1);
        if (t_lo > t_hi) return;  // no row of this chunk sees the tile (nothing to add)
    } else {
        t_lo = base;
        t_hi = min(a.T - 1, ((base + cnt - 1) / a.m + 1) * a.m + a.w - 2);
    }
    load_entries<D>(a, pooled, base, cnt, b, g, Ks, Vs);
    const int e0 = 2 * ty;
    float dk[2][4 * NC], dv[2][4 * NC];
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int c = 0; c < 4 * NC; ++c) dk[j][c] = dv[j][c] = 0.f;

    for (int hh = 0; hh < rg && t_lo <= t_hi; ++hh) {
        const int h = g * rg + hh;
        for (int rt = (t_lo / RT) * RT; rt <= t_hi; rt += RT) {
            const int nrow = min(RT, a.T - rt);
            __syncthreads();  // the previous row tile is consumed (and K, V are in place)
            for (int i = tid; i < RT * (D / 4); i += kTT) {
                const int r = i / (D / 4), c = 4 * (i % (D / 4));
                float4 q4 = make_float4(0.f, 0.f, 0.f, 0.f), d4 = q4;
                if (r < nrow) {
                    const size_t row = ((size_t)b * a.T + rt + r) * a.Hq + h;
                    q4 = ld4(a.qf + row * D + c);
                    q4.x *= a.scale; q4.y *= a.scale; q4.z *= a.scale; q4.w *= a.scale;
                    d4 = ld4(a.dof + row * D + c);
                }
                st4(Qs + r * LD + c, q4);
                st4(dOs + r * LD + c, d4);
            }
            for (int r = tid; r < RT; r += kTT) {
                const size_t row = ((size_t)b * a.T + rt + r) * a.Hq + h;
                lse_s[r] = r < nrow ? a.lse[row] : 0.f;
                dsum_s[r] = r < nrow ? a.dsum[row] : 0.f;
                Prow[r] = visible_blocks(rt + r + 1, a.m, a.w);
            }
            __syncthreads();
            float sc[2][4], dp[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int i = 0; i < 4; ++i) sc[j][i] = dp[j][i] = 0.f;
#pragma unroll 2
            for (int d = 0; d < D; d += 4) {
                const float4 k0 = ld4(Ks + e0 * LD + d), k1 = ld4(Ks + (e0 + 1) * LD + d);
                const float4 v0 = ld4(Vs + e0 * LD + d), v1 = ld4(Vs + (e0 + 1) * LD + d);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 q4 = ld4(Qs + (tx + 16 * i) * LD + d);
                    const float4 d4 = ld4(dOs + (tx + 16 * i) * LD + d);
                    sc[0][i] = dot4(k0, q4, sc[0][i]);
                    sc[1][i] = dot4(k1, q4, sc[1][i]);
                    dp[0][i] = dot4(v0, d4, dp[0][i]);
                    dp[1][i] = dot4(v1, d4, dp[1][i]);
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = tx + 16 * i, e = e0 + j;
                    const bool ok = r < nrow && e < cnt && sees(pooled, base + e, rt + r, Prow[r], a.m);
                    const float p = ok ? expf(sc[j][i] - lse_s[r]) : 0.f;
                    PT[e * (RT + 1) + r] = p;
                    dST[e * (RT + 1) + r] = p * (dp[j][i] - dsum_s[r]);
                }
            __syncthreads();
            for (int r = 0; r < nrow; ++r) {
                const float p0 = PT[e0 * (RT + 1) + r], p1 = PT[(e0 + 1) * (RT + 1) + r];
                const float s0 = dST[e0 * (RT + 1) + r], s1 = dST[(e0 + 1) * (RT + 1) + r];
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    const float4 d4 = ld4(dOs + r * LD + 64 * c + 4 * tx);
                    const float4 q4 = ld4(Qs + r * LD + 64 * c + 4 * tx);
                    axpy4(p0, d4, &dv[0][4 * c]);
                    axpy4(p1, d4, &dv[1][4 * c]);
                    axpy4(s0, q4, &dk[0][4 * c]);
                    axpy4(s1, q4, &dk[1][4 * c]);
                }
            }
        }
    }
    const size_t npool = (size_t)a.B * a.NB * a.G;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int e = e0 + j;
        if (e >= cnt) continue;
        const size_t r = pooled ? (((size_t)b * a.NB + base + e) * a.G + g) : (((size_t)b * a.T + base + e) * a.G + g);
        float* dko = pooled ? a.dE + r * D : a.dKf + r * D;
        float* dvo = pooled ? a.dE + (npool + r) * D : a.dv + r * D;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            float4 kv = make_float4(dk[j][4 * c], dk[j][4 * c + 1], dk[j][4 * c + 2], dk[j][4 * c + 3]);
            const float4 vv = make_float4(dv[j][4 * c], dv[j][4 * c + 1], dv[j][4 * c + 2], dv[j][4 * c + 3]);
            if (a.shared) {
                kv.x += vv.x; kv.y += vv.y; kv.z += vv.z; kv.w += vv.w;
            }
            if (pooled) {  // one chunk's share
                float* pk = dko + 64 * c + 4 * tx;
                atomicAdd(pk, kv.x); atomicAdd(pk + 1, kv.y); atomicAdd(pk + 2, kv.z); atomicAdd(pk + 3, kv.w);
                if (!a.shared) {
                    float* pv = dvo + 64 * c + 4 * tx;
                    atomicAdd(pv, vv.x); atomicAdd(pv + 1, vv.y); atomicAdd(pv + 2, vv.z); atomicAdd(pv + 3, vv.w);
                }
            } else {
                if (!a.shared) st4(dvo + 64 * c + 4 * tx, vv);
                st4(dko + 64 * c + 4 * tx, kv);
            }
        }
    }
}

template <int D>
cudaError_t tiled_attr() {
    static bool set[64] = {};  // per device
    const int dev_ = current_device();
    if (dev_ < 0 || !set[dev_]) {
        cudaError_t e = cudaFuncSetAttribute(row_pass_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)row_pass_smem<D>());
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(entry_pass_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)entry_pass_smem<D>());
        if (e != cudaSuccess) return e;
        if (dev_ >= 0) set[dev_] = true;
    }
    return cudaSuccess;
}

inline unsigned warps_grid(size_t warps) { return (unsigned)((warps + kWarpsPerCta - 1) / kWarpsPerCta); }

template <typename T, int NPL>
cudaError_t run_rows(const BwdArgs& a, cudaStream_t s) {
    const size_t nk = (size_t)a.B * a.NB * a.G, nr = (size_t)a.B * a.T * a.G, nq = (size_t)a.B * a.T * a.Hq;
    const dim3 blk(32 * kWarpsPerCta);
    finalise_kernel<T, NPL><<<warps_grid(nk + nr + nq), blk, 0, s>>>(a);
    constexpr int D = 32 * NPL;
    if constexpr (D == 64 || D == 128) {  // register-tiled passes
        cudaError_t e = tiled_attr<D>();
        if (e != cudaSuccess) return e;
        row_pass_kernel<D><<<dim3((a.T + RT - 1) / RT, a.Hq, a.B), kTT, row_pass_smem<D>(), s>>>(a);
        dq_tail_kernel<T, NPL><<<warps_grid(nq), blk, 0, s>>>(a);
        const int nchunk = (a.T + RT * kRowChunk - 1) / (RT * kRowChunk);
        const int tiles = (a.NB + ET - 1) / ET * nchunk + (a.T + ET - 1) / ET;
        // the pooled entries' gradients are sums over row chunks
        const size_t pooled = (size_t)a.S * a.B * a.NB * a.G * D;
        if (pooled && (e = cudaMemsetAsync(a.dE, 0, pooled * 4, s)) != cudaSuccess) return e;
        entry_pass_kernel<D><<<dim3(tiles, a.G, a.B), kTT, entry_pass_smem<D>(), s>>>(a);
    } else {
        row_lse_kernel<NPL><<<warps_grid(nq), blk, 0, s>>>(a);
        dq_kernel<T, NPL><<<warps_grid(nq), blk, 0, s>>>(a);
        dkv_kernel<NPL><<<warps_grid(nk + nr), blk, 0, s>>>(a);
    }
    key_bwd_kernel<T, NPL><<<warps_grid(nk + nr), blk, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t run_all(const BwdArgs& a, cudaStream_t s) {
    const size_t npool = (size_t)a.S * a.B * a.NB * a.G * a.D;
    const unsigned pg = (unsigned)std::min<size_t>((npool + 255) / 256, 148 * 16);
    if (npool) pool_fwd_kernel<T><<<std::max(pg, 1u), 256, 0, s>>>(a);
    cudaError_t e = cudaSuccess;
    switch (a.D / 32) {
        case 1: e = run_rows<T, 1>(a, s); break;
        case 2: e = run_rows<T, 2>(a, s); break;
        case 4: e = run_rows<T, 4>(a, s); break;
        case 8: e = run_rows<T, 8>(a, s); break;
        case 16: e = run_rows<T, 16>(a, s); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    if (npool) pool_bwd_kernel<T><<<std::max(pg, 1u), 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool backward_supported(int D) { return D == 32 || D == 64 || D == 128 || D == 256 || D == 512; }

size_t backward_scratch_floats(int S, int B, int T, int Hq, int G, int D, int m) {
    const size_t NB = (size_t)(T / m);
    const size_t pooled = (size_t)S * B * NB * G * D;
    const size_t raw = (size_t)B * T * G * D, rows = (size_t)B * T * Hq;
    // Ef, dE (both series), Pk, Kf, dKf, vf (GQA), qf, dof, lse, dsum
    return 2 * pooled + (size_t)B * NB * G * D + (S == 2 ? 3 : 2) * raw + 2 * rows * D + 2 * rows;
}

cudaError_t launch_backward(const BwdArgs& a, cudaStream_t s) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    return a.dtype == LBCA_BF16 ? run_all<__nv_bfloat16>(a, s) : run_all<float>(a, s);
}

}  // namespace lbca
