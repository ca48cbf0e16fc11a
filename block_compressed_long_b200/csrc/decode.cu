// decode.cu -- split-KV decode over pooled entries plus the raw window.
//
// One query per sequence at position t = L - 1 attends, in one softmax, to the
// visible pooled entries j < P(L) and the raw tokens s in [P(L) m, t], plus an
// optional sink logit that only enters the denominator (mSeek README, "How
// LBCA works", step 4; HCA page, "What is implemented"; CSA page, "What is
// implemented": Eqs 18-19, Eq 27, the -i output rotation of the shared form).
//
// B200 mapping (HBM-bound streaming):
//   grid = (split, head group, sequence).  A CTA owns R query heads of one kv
//   head and a chunk of the visible entry list.  Thread 0 issues bulk async
//   copies (cp.async.bulk, the non-tensor TMA path, no multicast) of the
//   chunk's pooled rows and raw ring rows straight into shared memory, with
//   completion on an mbarrier, while all threads prepare the queries (RMSNorm,
//   RoPE at t, scale folded with log2 e).  Groups of D/16 lanes then take one
//   entry each (16 dims per lane, conflict-free 16-byte shared loads), two
//   entries per step with one online-softmax rescale.  Groups merge through
//   shared memory; each CTA writes its (max, sum, unnormalised output) partial
//   and the last CTA of its (sequence, head group), found with one atomic
//   counter, merges the partials, adds the sink and writes the output.  The
//   counter is reset by that CTA, so the workspace stays zeroed between calls.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace lbca {
namespace {

constexpr int kThreads = 128;
constexpr int kMinChunk = 16;

struct Layout {
    size_t qs, cs, flag, stage, red_o, red_ml, total;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline Layout layout(int D, int R, int chunk, int esize, int shared) {
    const int NG = 4 * 32 / (D / 16);
    Layout l;
    l.qs = 16;
    l.cs = l.qs + (size_t)R * D * 4;
    l.flag = l.cs + (size_t)(D / 2) * 8;
    l.stage = align_up(l.flag + 16, 128);
    l.red_o = align_up(l.stage + (size_t)chunk * D * esize * (shared ? 1 : 2), 16);
    l.red_ml = l.red_o + (size_t)NG * R * D * 4;
    l.total = l.red_ml + (size_t)NG * R * 2 * 4;
    return l;
}

template <typename T>
__device__ __forceinline__ void store2(T* p, float a, float b);
template <> __device__ __forceinline__ void store2<float>(float* p, float a, float b) {
    *reinterpret_cast<float2*>(p) = make_float2(a, b);
}
template <> __device__ __forceinline__ void store2<__nv_bfloat16>(__nv_bfloat16* p, float a, float b) {
    *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(a, b);
}

// Shared form: a raw window row, held as 16 dims per lane over the LG lanes of
// an entry group (lane gl holds dims (c LG + gl) VEC + i), is finalised as it
// is read -- RMSNorm over the whole row (when on), then RoPE of the rotated
// dims at the token's position `pos` -- in f32, so that the entry the output
// averages carries no rounding beyond its input's.  Every lane of the warp
// calls it (the row sum crosses lanes); `raw` is uniform per entry group.
template <typename T, int D, int LG, int VEC>
__device__ __forceinline__ void finalise_raw16(float (&x)[16], bool raw, int64_t pos, int gl, const DecodeArgs& a) {
    constexpr int NCH = 16 / VEC;
    if (a.rmsnorm) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) ss = fmaf(x[i], x[i], ss);
#pragma unroll
        for (int off = LG / 2; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (raw) {
            const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
            const T* gm = static_cast<const T*>(a.gamma_kv);
#pragma unroll
            for (int c = 0; c < NCH; ++c)
#pragma unroll
                for (int i = 0; i < VEC; ++i)
                    x[c * VEC + i] *= inv * (gm ? to_f<T>(gm[(c * LG + gl) * VEC + i]) : 1.0f);
        }
    }
    if (raw && a.rho) {
        const int base = D - a.rho;
#pragma unroll
        for (int c = 0; c < NCH; ++c)
#pragma unroll
            for (int i = 0; i < VEC; i += 2) {
                const int d = (c * LG + gl) * VEC + i;
                if (d >= base) rotate_pair(x[c * VEC + i], x[c * VEC + i + 1], rope_cs(pos, (d - base) >> 1, a.rope_step));
            }
    }
}

template <typename T, int D, int R>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeArgs a) {
    constexpr int VEC = Vec<T>::N;
    constexpr int LG = D / 16;        // lanes per entry
    constexpr int NCH = 16 / VEC;     // 16-byte chunks per lane
    constexpr int GPW = 32 / LG;      // entry groups per warp
    constexpr int NG = 4 * GPW;       // entry groups per CTA
    constexpr uint32_t ROW = D * sizeof(T);

    extern __shared__ __align__(128) unsigned char smem[];
    const Layout lay = layout(D, R, a.chunk, sizeof(T), a.shared);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
    float* qs = reinterpret_cast<float*>(smem + lay.qs);
    float2* cs = reinterpret_cast<float2*>(smem + lay.cs);
    int* flag = reinterpret_cast<int*>(smem + lay.flag);
    T* kbuf = reinterpret_cast<T*>(smem + lay.stage);
    T* vbuf = a.shared ? kbuf : kbuf + (size_t)a.chunk * D;
    float* red_o = reinterpret_cast<float*>(smem + lay.red_o);
    float* red_ml = reinterpret_cast<float*>(smem + lay.red_ml);

    const int split = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = a.Hq / a.G;
    const int h0 = hg * R;
    const int g = h0 / r;

    // ---- visible set of this sequence (block-aligned partition) ----
    const int L = a.seq_lens[b];
    const int t = L - 1;
    const int P = visible_blocks(L, a.m, a.w);
    const int s0 = P * a.m;
    int n_vis = L > 0 ? P + (L - s0) : 0;
    if (P > a.max_blocks || L - s0 > a.R) {  // cache cannot hold this state
        if (split == 0 && hg == 0 && tid == 0) set_status(a.status, LBCA_ERR_CAPACITY);
        n_vis = 0;
    }
    int nsp = max(1, (n_vis + a.chunk - 1) / a.chunk);
    if (nsp > a.n_split) {
        if (split == 0 && hg == 0 && tid == 0) set_status(a.status, LBCA_ERR_CAPACITY);
        nsp = a.n_split;
    }
    if (split >= nsp) return;  // uniform per CTA
    const int e0 = split * a.chunk;
    const int e1 = min(n_vis, e0 + a.chunk);
    const int ne = max(0, e1 - e0);

    // ---- stage the chunk: pooled rows, then raw ring rows (at most one wrap) ----
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (tid == 0 && ne > 0) {
        mbar_arrive_expect_tx(bar, (uint32_t)ne * ROW * (a.shared ? 1u : 2u));
        const size_t pool_head = ((size_t)b * a.G + g) * a.max_blocks;
        const size_t ring_head = ((size_t)b * a.G + g) * a.R;
        int e = e0, row = 0;
        if (e < P) {
            const int n = min(e1, P) - e;
            bulk_g2s(kbuf, static_cast<const T*>(a.pooled_k) + (pool_head + checked_rows(e, n, a.max_blocks, a.status)) * D, n * ROW, bar);
            if (!a.shared)
                bulk_g2s(vbuf, static_cast<const T*>(a.pooled_v) + (pool_head + checked_rows(e, n, a.max_blocks, a.status)) * D, n * ROW, bar);
            e += n;
            row += n;
        }
        while (e < e1) {
            const int slot = (s0 + (e - P)) % a.R;
            const int n = min(e1 - e, a.R - slot);
            bulk_g2s(kbuf + (size_t)row * D, static_cast<const T*>(a.ring_k) + (ring_head + checked_rows(slot, n, a.R, a.status)) * D,
                     n * ROW, bar);
            if (!a.shared)
                bulk_g2s(vbuf + (size_t)row * D,
                         static_cast<const T*>(a.ring_v) + (ring_head + checked_rows(slot, n, a.R, a.status)) * D, n * ROW, bar);
            e += n;
            row += n;
        }
    }

    // ---- query prep overlaps the copies: RMSNorm, RoPE at t, log2-domain scale ----
    for (int k = tid; k < a.rho / 2; k += kThreads) cs[k] = rope_cs((int64_t)t, k, a.rope_step);
    for (int idx = tid; idx < R * D / VEC; idx += kThreads) {
        const int h = idx / (D / VEC), c = idx % (D / VEC);
        float v[VEC];
        ld16(static_cast<const T*>(a.q) + ((size_t)b * a.Hq + h0 + h) * D + c * VEC, v);
#pragma unroll
        for (int i = 0; i < VEC; ++i) qs[h * D + c * VEC + i] = v[i];
    }
    __syncthreads();
    if (a.rmsnorm) {
        for (int h = warp; h < R; h += kThreads / 32) {
            float ss = 0.f;
            for (int d = lane; d < D; d += 32) ss += qs[h * D + d] * qs[h * D + d];
#pragma unroll
            for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
            const T* gm = static_cast<const T*>(a.gamma_q);
            for (int d = lane; d < D; d += 32) qs[h * D + d] *= inv * (gm ? to_f<T>(gm[d]) : 1.0f);
        }
        __syncthreads();
    }
    for (int idx = tid; idx < R * (a.rho / 2); idx += kThreads) {
        const int h = idx / (a.rho / 2), k = idx % (a.rho / 2);
        const int d = D - a.rho + 2 * k;
        rotate_pair(qs[h * D + d], qs[h * D + d + 1], cs[k]);
    }
    __syncthreads();

    const int grp = warp * GPW + lane / LG;
    const int gl = lane % LG;
    const float qscale = a.scale * kLog2e;
    float qr[R][16];
#pragma unroll
    for (int h = 0; h < R; ++h)
#pragma unroll
        for (int c = 0; c < NCH; ++c)
#pragma unroll
            for (int i = 0; i < VEC; ++i) qr[h][c * VEC + i] = qs[h * D + (c * LG + gl) * VEC + i] * qscale;

    bool ok = true;
    if (ne > 0) ok = mbar_wait(bar, 0);
    ok = __syncthreads_and(ok);
    int n_use = ne;
    if (!ok) {
        if (tid == 0) {
            set_status(a.status, LBCA_ERR_TIMEOUT);
            mbar_wait(bar, 0);  // give copies in flight a last bounded chance to land
        }
        n_use = 0;
    }

    // ---- stream the chunk: two entries per group per step ----
    float mx[R], ls[R], o[R][16];
#pragma unroll
    for (int h = 0; h < R; ++h) {
        mx[h] = kNegInf;
        ls[h] = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) o[h][i] = 0.f;
    }
    for (int eb = warp * GPW; eb < n_use; eb += 2 * NG) {
        const int ea = eb + lane / LG, ebb = ea + NG;
        const bool va = ea < n_use, vb = ebb < n_use;
        const T* ka = kbuf + (size_t)(va ? ea : 0) * D;
        const T* kb = kbuf + (size_t)(vb ? ebb : 0) * D;
        float kfa[16], kfb[16];
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            float t0[VEC], t1[VEC];
            ld16(ka + (c * LG + gl) * VEC, t0);
            ld16(kb + (c * LG + gl) * VEC, t1);
#pragma unroll
            for (int i = 0; i < VEC; ++i) { kfa[c * VEC + i] = t0[i]; kfb[c * VEC + i] = t1[i]; }
        }
        if (a.shared) {  // rows past the pooled ones are raw window entries
            const int ia = e0 + ea, ib = e0 + ebb;
            finalise_raw16<T, D, LG, VEC>(kfa, va && ia >= P, (int64_t)s0 + (ia - P), gl, a);
            finalise_raw16<T, D, LG, VEC>(kfb, vb && ib >= P, (int64_t)s0 + (ib - P), gl, a);
        }
        float sa[R], sb[R];
#pragma unroll
        for (int h = 0; h < R; ++h) {
            float x = 0.f, y = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) { x = fmaf(qr[h][i], kfa[i], x); y = fmaf(qr[h][i], kfb[i], y); }
            sa[h] = x;
            sb[h] = y;
        }
#pragma unroll
        for (int off = LG / 2; off; off >>= 1)
#pragma unroll
            for (int h = 0; h < R; ++h) {
                sa[h] += __shfl_xor_sync(0xffffffffu, sa[h], off);
                sb[h] += __shfl_xor_sync(0xffffffffu, sb[h], off);
            }
        if (!va) continue;  // no shuffles below
        float vfa[16], vfb[16];
        if (a.shared) {  // the (finalised) entry is its own value
#pragma unroll
            for (int i = 0; i < 16; ++i) { vfa[i] = kfa[i]; vfb[i] = kfb[i]; }
        } else {
            const T* vra = vbuf + (size_t)ea * D;
            const T* vrb = vbuf + (size_t)(vb ? ebb : ea) * D;
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                float t0[VEC], t1[VEC];
                ld16(vra + (c * LG + gl) * VEC, t0);
                ld16(vrb + (c * LG + gl) * VEC, t1);
#pragma unroll
                for (int i = 0; i < VEC; ++i) { vfa[c * VEC + i] = t0[i]; vfb[c * VEC + i] = t1[i]; }
            }
        }
#pragma unroll
        for (int h = 0; h < R; ++h) {
            const float sbh = vb ? sb[h] : kNegInf;
            const float mn = fmaxf(mx[h], fmaxf(sa[h], sbh));
            const float rr = ex2(mx[h] - mn);
            const float pa = ex2(sa[h] - mn);
            const float pb = ex2(sbh - mn);
            ls[h] = fmaf(ls[h], rr, pa + pb);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[h][i] = fmaf(o[h][i], rr, fmaf(pa, vfa[i], pb * vfb[i]));
            mx[h] = mn;
        }
    }

    // ---- merge the entry groups of this CTA ----
#pragma unroll
    for (int h = 0; h < R; ++h) {
#pragma unroll
        for (int c = 0; c < NCH; ++c)
#pragma unroll
            for (int i = 0; i < VEC; ++i)
                red_o[((size_t)grp * R + h) * D + (c * LG + gl) * VEC + i] = o[h][c * VEC + i];
        if (gl == 0) {
            red_ml[(grp * R + h) * 2] = mx[h];
            red_ml[(grp * R + h) * 2 + 1] = ls[h];
        }
    }
    __syncthreads();

    const float* sink = a.sink;
    auto finalise = [&](int h, int d, float o0, float o1, float M, float Ls) {
        float den = Ls;
        if (sink) den += (M == kNegInf) ? 1.0f : ex2(sink[h0 + h] * kLog2e - M);
        float v0 = den > 0.f ? o0 / den : 0.f, v1 = den > 0.f ? o1 / den : 0.f;
        if (a.shared && a.rho && d >= D - a.rho) {
            const float2 c = cs[(d - (D - a.rho)) >> 1];
            rotate_pair(v0, v1, make_float2(c.x, -c.y));
        }
        store2<T>(static_cast<T*>(a.out) + ((size_t)b * a.Hq + h0 + h) * D + d, v0, v1);
    };

    for (int idx = tid; idx < R * D / 2; idx += kThreads) {
        const int h = idx / (D / 2), d = (idx % (D / 2)) * 2;
        float M = kNegInf;
        for (int q = 0; q < NG; ++q) M = fmaxf(M, red_ml[(q * R + h) * 2]);
        float Ls = 0.f, o0 = 0.f, o1 = 0.f;
        if (M != kNegInf) {
            for (int q = 0; q < NG; ++q) {
                const float f = ex2(red_ml[(q * R + h) * 2] - M);
                Ls = fmaf(red_ml[(q * R + h) * 2 + 1], f, Ls);
                o0 = fmaf(red_o[((size_t)q * R + h) * D + d], f, o0);
                o1 = fmaf(red_o[((size_t)q * R + h) * D + d + 1], f, o1);
            }
        }
        if (nsp == 1) {
            finalise(h, d, o0, o1, M, Ls);
        } else {
            const size_t pi = ((size_t)b * a.Hq + h0 + h) * a.n_split + split;
            *reinterpret_cast<float2*>(a.part_o + pi * D + d) = make_float2(o0, o1);
            if (d == 0) *reinterpret_cast<float2*>(a.part_ml + pi * 2) = make_float2(M, Ls);
        }
    }
    if (nsp == 1) return;

    // ---- last CTA of this (sequence, head group) merges the split partials ----
    __threadfence();
    __syncthreads();
    uint32_t* ctr = a.counters + (size_t)b * (a.Hq / R) + hg;
    if (tid == 0) *flag = (atomicAdd(ctr, 1u) == (uint32_t)(nsp - 1));
    __syncthreads();
    if (!*flag) return;
    __threadfence();
    // split weights 2^(m_s - M) per head, staged in shared memory (the group
    // reduction buffers are free now): all partial statistics load at once
    float* wsm = red_o;   // [nsp][R] (m, l) pairs, then (weight, l)
    float* mh = red_ml;   // [R] max, [R, 2R) denominator
    for (int idx = tid; idx < nsp * R; idx += kThreads) {
        const int sp = idx / R, h = idx % R;
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(
            a.part_ml + (((size_t)b * a.Hq + h0 + h) * a.n_split + sp) * 2));
        wsm[2 * idx] = ml.x;
        wsm[2 * idx + 1] = ml.y;
    }
    __syncthreads();
    if (warp < R) {
        const int h = warp;
        float M = kNegInf;
        for (int sp = lane; sp < nsp; sp += 32) M = fmaxf(M, wsm[2 * (sp * R + h)]);
#pragma unroll
        for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float Ls = 0.f;
        for (int sp = lane; sp < nsp; sp += 32) {
            const float f = M == kNegInf ? 0.f : ex2(wsm[2 * (sp * R + h)] - M);
            wsm[2 * (sp * R + h)] = f;
            Ls = fmaf(f, wsm[2 * (sp * R + h) + 1], Ls);
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, off);
        if (lane == 0) {
            mh[h] = M;
            mh[R + h] = Ls;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < R * D / 2; idx += kThreads) {
        const int h = idx / (D / 2), d = (idx % (D / 2)) * 2;
        const float* po = a.part_o + ((size_t)b * a.Hq + h0 + h) * a.n_split * D + d;
        float o0 = 0.f, o1 = 0.f;
#pragma unroll 8
        for (int sp = 0; sp < nsp; ++sp) {
            const float f = wsm[2 * (sp * R + h)];
            const float2 ov = __ldcg(reinterpret_cast<const float2*>(po + (size_t)sp * D));
            o0 = fmaf(ov.x, f, o0);
            o1 = fmaf(ov.y, f, o1);
        }
        finalise(h, d, o0, o1, mh[h], mh[R + h]);
    }
    if (tid == 0) *ctr = 0u;
}

template <typename T, int D, int R>
cudaError_t launch_one(const DecodeArgs& a, size_t smem, cudaStream_t s) {
    static bool attr_set[64] = {};  // per device
    const int dev_ = current_device();
    if (dev_ < 0 || !attr_set[dev_]) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<T, D, R>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return e;
        if (dev_ >= 0) attr_set[dev_] = true;
    }
    dim3 grid(a.n_split, a.Hq / R, a.B);
    decode_kernel<T, D, R><<<grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t dispatch_r(const DecodeArgs& a, size_t smem, cudaStream_t s) {
    switch (a.heads_per_cta) {
        case 1: return launch_one<T, D, 1>(a, smem, s);
        case 2: return launch_one<T, D, 2>(a, smem, s);
        case 3: return launch_one<T, D, 3>(a, smem, s);
        case 4: return launch_one<T, D, 4>(a, smem, s);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t dispatch_d(const DecodeArgs& a, size_t smem, cudaStream_t s) {
    switch (a.D) {
        case 16: return dispatch_r<T, 16>(a, smem, s);
        case 32: return dispatch_r<T, 32>(a, smem, s);
        case 64: return dispatch_r<T, 64>(a, smem, s);
        case 128: return dispatch_r<T, 128>(a, smem, s);
        case 256: return dispatch_r<T, 256>(a, smem, s);
        case 512: return dispatch_r<T, 512>(a, smem, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

DecodePlan plan_decode(int dtype, int B, int Hq, int G, int D, int m, int w, int shared, int max_ctx) {
    DecodePlan p{};
    p.ok = false;
    if (D != 16 && D != 32 && D != 64 && D != 128 && D != 256 && D != 512) return p;
    const int r = Hq / G;
    int R = 1;
    for (int c : {4, 3, 2, 1})
        if (r % c == 0) { R = c; break; }
    const int esize = dtype == LBCA_BF16 ? 2 : 4;
    if (max_ctx < 1) max_ctx = 1;
    const int P = max_ctx - w > 0 ? (max_ctx - w) / m : 0;
    const long long vis_bound = (long long)P + w + m - 1;
    const int max_vis = (int)std::min<long long>(max_ctx, vis_bound);
    const size_t row_bytes = (size_t)D * esize * (shared ? 1 : 2);
    int cmax = 16;
    while (cmax * 2 <= 256 && (size_t)(cmax * 2) * row_bytes <= 64 * 1024) cmax *= 2;
    const long long groups = (long long)B * (Hq / R);
    int chunk = kMinChunk;
    for (int c = cmax; c >= kMinChunk; c /= 2) {
        if (groups * ((max_vis + c - 1) / c) >= 148) { chunk = c; break; }  // one wave of SMs
    }
    p.heads_per_cta = R;
    p.chunk = chunk;
    p.n_split = std::max(1, (max_vis + chunk - 1) / chunk);
    p.part_o_elems = (size_t)B * Hq * p.n_split * D;
    p.part_ml_elems = (size_t)B * Hq * p.n_split * 2;
    p.counter_elems = (size_t)B * (Hq / R);
    p.smem_bytes = layout(D, R, chunk, esize, shared).total;
    // the merge stages 2 floats per (split, head) in the group-reduction buffer
    p.ok = p.smem_bytes <= 200 * 1024 && p.n_split * 2 <= (2048 / D) * D;
    return p;
}

size_t decode_workspace_bytes(const DecodePlan& p) {
    return align_up(p.part_o_elems * 4, 256) + align_up(p.part_ml_elems * 4, 256) +
           align_up(p.counter_elems * 4, 256);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
    if (a.B == 0) return cudaSuccess;
    const size_t smem = layout(a.D, a.heads_per_cta, a.chunk, a.dtype == LBCA_BF16 ? 2 : 4, a.shared).total;
    if (a.dtype == LBCA_BF16) return dispatch_d<__nv_bfloat16>(a, smem, s);
    return dispatch_d<float>(a, smem, s);
}

}  // namespace lbca
