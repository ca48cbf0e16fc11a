// decode_step.cu -- one serving step in one launch: append the new raw token
// and decode its query, with the split merge done inside a thread-block
// cluster over distributed shared memory.
//
// What is computed is lbca_append followed by lbca_decode (mSeek README, "How
// LBCA works", steps 2-5; HCA page and CSA page, "What is implemented"): the
// query at t = L_old sees pooled entries j < P(L_old + 1) and raw tokens
// [P m, t].  With n_win >= 1 the block the new token may complete is never
// visible to the same step (it becomes visible n_win tokens later), so the
// append work (running pooling softmax, block finalisation, ring write) is
// independent of this step's attention and runs after it, off the critical
// path.  The newest raw row itself is finalised in shared memory by the CTA
// that needs it instead of being read back from the ring.
//
// B200 mapping: grid (CS, head groups, sequences) with cluster (CS, 1, 1).  The
// CS CTAs of a cluster split one (sequence, head group)'s visible entries
// evenly, stream them through a two-stage shared-memory ring filled by bulk
// async copies (cp.async.bulk, non-multicast), and publish their (max, sum,
// unnormalised output) partials in shared memory; after a cluster barrier
// each CTA merges a slice of the head dims by reading its peers' partials over
// DSMEM.  No global partials, fences or atomics sit between the last entry and
// the output.  The CTA that arrives last for a sequence advances seq_lens.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"
#include "decode_common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace lbca {
namespace {

constexpr int kThreads = 128;

struct StepLayout {
    size_t bars, misc, qs, cs, newk, newv, wred_o, wred_ml, recv_o, recv_ml, stage, total;
};

__host__ __device__ inline size_t al(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kWarps = kThreads / 32;

__host__ __device__ inline StepLayout step_layout(int D, int R, int SE, int esize, int shared, int CS) {
    StepLayout l;
    l.bars = 0;
    l.misc = 16;                                   // broadcast of t + block_sum scratch
    l.qs = 64;
    l.cs = l.qs + (size_t)R * D * 4;
    l.newk = al(l.cs + (size_t)(D / 2) * 8, 16);
    l.newv = l.newk + (size_t)D * esize;
    l.wred_o = al(l.newv + (size_t)D * esize, 16);
    l.wred_ml = l.wred_o + (size_t)kWarps * R * D * 4;
    l.recv_o = al(l.wred_ml + (size_t)kWarps * R * 2 * 4, 16);
    l.recv_ml = l.recv_o + (size_t)R * D * 4;      // CS slices of D / CS dims
    l.stage = al(l.recv_ml + (size_t)CS * R * 2 * 4, 128);
    l.total = l.stage + 2 * (size_t)SE * D * esize * (shared ? 1 : 2);
    return l;
}

// Block-wide sum over kThreads threads (every thread must call it).
__device__ __forceinline__ float block_sum(float v, float* scratch) {
#pragma unroll
    for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) s += scratch[i];
    __syncthreads();
    return s;
}

template <typename T, int D, int R>
__global__ void __launch_bounds__(kThreads) decode_step_kernel(const StepArgs a) {
    constexpr int VEC = Vec<T>::N;
    constexpr int LG = D / 16;       // lanes per entry
    constexpr int NCH = 16 / VEC;    // 16-byte chunks per lane
    constexpr int GPW = 32 / LG;     // entry groups per warp
    constexpr int NG = kWarps * GPW; // entry groups per CTA
    constexpr uint32_t ROW = D * sizeof(T);

    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ __align__(128) unsigned char smem[];
    const int CS = a.CS;
    const StepLayout lay = step_layout(D, R, a.SE, sizeof(T), a.shared, CS);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + lay.bars);
    int* tsh = reinterpret_cast<int*>(smem + lay.misc);
    float* scratch = reinterpret_cast<float*>(smem + lay.misc + 16);
    float* qs = reinterpret_cast<float*>(smem + lay.qs);
    float2* cs = reinterpret_cast<float2*>(smem + lay.cs);
    T* newk = reinterpret_cast<T*>(smem + lay.newk);
    T* newv = reinterpret_cast<T*>(smem + lay.newv);
    float* wred_o = reinterpret_cast<float*>(smem + lay.wred_o);
    float* wred_ml = reinterpret_cast<float*>(smem + lay.wred_ml);
    float* recv_o = reinterpret_cast<float*>(smem + lay.recv_o);
    float* recv_ml = reinterpret_cast<float*>(smem + lay.recv_ml);
    T* kst = reinterpret_cast<T*>(smem + lay.stage);        // [2][SE][D]
    T* vst = a.shared ? kst : kst + 2 * (size_t)a.SE * D;    // [2][SE][D]

    const int rank = (int)cluster.block_rank();
    const int hg = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = a.Hq / a.G;
    const int h0 = hg * R;
    const int g = h0 / r;
    const int GD = a.G * D;
    const int DS = D / CS;  // dims this CTA finalises

    // ---- the open block's running pooling state (this cache's; read before the
    // preceding kernel completes when launched with programmatic dependence) ----
    const bool app = rank == 0 && h0 % r == 0;  // the CTA that appends for (sequence, kv head)
    const bool pair_owner = tid < D / 2;
    constexpr int QV = (R * D / VEC + kThreads - 1) / kThreads;
    uint4 qv[QV];
    const size_t tok = (size_t)b * GD + (size_t)g * D + 2 * tid;  // this thread's pair of the new token
    typename Pair<T>::Raw kraw{}, vraw{}, zraw[2]{};
    float2 am[2], al_[2], aa[2];  // running pooling state of the open block
    if (pair_owner && app) {
#pragma unroll
        for (int s = 0; s < 2; ++s) {  // series: key (or shared entry), value
            if (s >= a.S) break;
            const float* st = a.state + (((size_t)b * a.S + s) * 3) * GD + (size_t)g * D + 2 * tid;
            am[s] = *reinterpret_cast<const float2*>(st);
            al_[s] = *reinterpret_cast<const float2*>(st + GD);
            aa[s] = *reinterpret_cast<const float2*>(st + 2 * GD);
        }
    }

    // ---- the step: token t = L_old joins, the query sits at t ----
    if (tid == 0) {
        *tsh = a.seq_lens[b];  // read once, broadcast
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_barrier_init();
    }
    __syncthreads();
    const int t = *tsh;
    const int L = t + 1;
    const int P = visible_blocks(L, a.m, a.w);
    const int s0 = P * a.m;
    int n_vis = P + (L - s0);
    if (P > a.max_blocks || L - s0 > a.R) {
        if (rank == 0 && hg == 0 && tid == 0) set_status(a.status, LBCA_ERR_CAPACITY);
        n_vis = 0;
    }
    const int chunk = (n_vis + CS - 1) / CS;
    const int e0 = min(n_vis, rank * chunk);
    const int e1 = min(n_vis, e0 + chunk);
    const int ne = e1 - e0;
    const int nst = (ne + a.SE - 1) / a.SE;
    const int newest = n_vis - 1;  // the raw token t itself: built in shared memory

    auto issue = [&](int st) {  // thread 0 only: bulk copies of stage st into buffer st & 1
        const int b0 = e0 + st * a.SE, b1 = min(e1, b0 + a.SE);
        T* kd = kst + (size_t)(st & 1) * a.SE * D;
        T* vd = vst + (size_t)(st & 1) * a.SE * D;
        const int c1 = min(b1, newest);  // rows [b0, c1) come from memory
        const uint32_t rows = c1 > b0 ? (uint32_t)(c1 - b0) : 0u;
        mbar_arrive_expect_tx(&bars[st & 1], rows * ROW * (a.shared ? 1u : 2u));
        const size_t pool_head = ((size_t)b * a.G + g) * a.max_blocks;
        const size_t ring_head = ((size_t)b * a.G + g) * a.R;
        int e = b0, row = 0;
        if (e < c1 && e < P) {
            const int n = min(c1, P) - e;
            bulk_g2s(kd, static_cast<const T*>(a.pooled_k) + (pool_head + checked_rows(e, n, a.max_blocks, a.status)) * D, n * ROW, &bars[st & 1]);
            if (!a.shared)
                bulk_g2s(vd, static_cast<const T*>(a.pooled_v) + (pool_head + checked_rows(e, n, a.max_blocks, a.status)) * D, n * ROW, &bars[st & 1]);
            e += n;
            row += n;
        }
        while (e < c1) {
            const int slot = (s0 + (e - P)) % a.R;
            const int n = min(c1 - e, a.R - slot);
            bulk_g2s(kd + (size_t)row * D, static_cast<const T*>(a.ring_k) + (ring_head + checked_rows(slot, n, a.R, a.status)) * D, n * ROW,
                     &bars[st & 1]);
            if (!a.shared)
                bulk_g2s(vd + (size_t)row * D, static_cast<const T*>(a.ring_v) + (ring_head + checked_rows(slot, n, a.R, a.status)) * D, n * ROW,
                         &bars[st & 1]);
            e += n;
            row += n;
        }
    };

    if (tid == 0) {
        if (nst > 0) issue(0);
        if (nst > 1) issue(1);
    }

    // ---- the step's own inputs (the query and the new token) may come from the
    // preceding kernel: everything above reads only this cache ----
    griddep_wait();
    if (tid == 0) {
        // Every CTA of the sequence has read its length once it has arrived
        // here, so the last to arrive may advance it (latency hidden behind
        // the copies).
        const uint32_t total = (uint32_t)(CS * (a.Hq / R));
        if (atomicAdd(&a.arrive[b], 1u) == total - 1) {
            a.seq_lens[b] = L;
            a.arrive[b] = 0u;
        }
    }
#pragma unroll
    for (int j = 0; j < QV; ++j) {
        const int idx = tid + j * kThreads;
        if (idx < R * D / VEC)
            qv[j] = *reinterpret_cast<const uint4*>(static_cast<const T*>(a.q) + ((size_t)b * a.Hq + h0 + idx / (D / VEC)) * D +
                                                    (idx % (D / VEC)) * VEC);
    }
    if (pair_owner) {
        kraw = Pair<T>::load(static_cast<const T*>(a.k) + tok);
        if (!a.shared) vraw = Pair<T>::load(static_cast<const T*>(a.v) + tok);
        if (app) {
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                if (s >= a.S) break;
                zraw[s] = Pair<T>::load(static_cast<const T*>(s == 0 ? a.zk : a.zv) + tok);
            }
        }
    }

    // ---- the appending CTA: B_pos row of the new token's offset in its block ----
    const int ai = t % a.m, aj = t / a.m;
    float2 abp[2];
    if (app && pair_owner)
#pragma unroll
        for (int s = 0; s < 2; ++s)
            if (s < a.S) abp[s] = get2(static_cast<const T*>(s == 0 ? a.bpk : a.bpv) + (size_t)ai * GD + (size_t)g * D + 2 * tid);

    // ---- query prep and the newest raw row, overlapping the copies ----
    for (int k = tid; k < a.rho / 2; k += kThreads) cs[k] = rope_cs((int64_t)t, k, a.rope_step);
#pragma unroll
    for (int j = 0; j < QV; ++j) {
        const int idx = tid + j * kThreads;
        if (idx < R * D / VEC) {
            float v[VEC];
            unpack16<T>(qv[j], v);
#pragma unroll
            for (int i = 0; i < VEC; ++i) qs[(idx / (D / VEC)) * D + (idx % (D / VEC)) * VEC + i] = v[i];
        }
    }
    float2 kraw_f = make_float2(0.f, 0.f);  // the new raw key before RMSNorm / RoPE (pooled raw)
    float2 kx = make_float2(0.f, 0.f), vx = kx;
    if (pair_owner) {
        kx = Pair<T>::cvt(kraw);
        kraw_f = kx;
        if (!a.shared) vx = Pair<T>::cvt(vraw);
    }
    __syncthreads();  // cs, qs ready
    {
        const float ss = a.rmsnorm ? block_sum(pair_owner ? kx.x * kx.x + kx.y * kx.y : 0.f, scratch) : 0.f;
        if (pair_owner) {
            if (a.rmsnorm) {
                const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
                const T* gm = static_cast<const T*>(a.gamma_kv);
                kx.x *= inv * (gm ? to_f<T>(gm[2 * tid]) : 1.f);
                kx.y *= inv * (gm ? to_f<T>(gm[2 * tid + 1]) : 1.f);
            }
            if (a.rho && 2 * tid >= D - a.rho) rotate_pair(kx.x, kx.y, cs[(2 * tid - (D - a.rho)) >> 1]);
            put2<T>(newk + 2 * tid, kx.x, kx.y);
            if (!a.shared) put2<T>(newv + 2 * tid, vx.x, vx.y);
        }
    }
    if (a.rmsnorm) {
        for (int h = warp; h < R; h += kWarps) {
            float ss = 0.f;
            for (int d = lane; d < D; d += 32) ss += qs[h * D + d] * qs[h * D + d];
#pragma unroll
            for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
            const T* gm = static_cast<const T*>(a.gamma_q);
            for (int d = lane; d < D; d += 32) qs[h * D + d] *= inv * (gm ? to_f<T>(gm[d]) : 1.0f);
        }
    }
    __syncthreads();
    for (int idx = tid; idx < R * (a.rho / 2); idx += kThreads) {
        const int h = idx / (a.rho / 2), k = idx % (a.rho / 2);
        const int d = D - a.rho + 2 * k;
        rotate_pair(qs[h * D + d], qs[h * D + d + 1], cs[k]);
    }
    __syncthreads();

    // ---- append the new token (one CTA per (sequence, kv head)) while the copies
    // land: running pooling softmax, block finalisation, ring write.  Nothing
    // it writes is visible to this step (the ring slot of t holds token t - R,
    // the block it may complete becomes visible n_win tokens later).
    if (app) {
        const bool complete = ai == a.m - 1;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            if (s >= a.S) break;
            const bool key = s == 0;
            float mxs[2] = {0.f, 0.f}, lss[2] = {1.f, 1.f}, acs[2] = {0.f, 0.f};
            if (pair_owner) {
                const float2 xs = key ? kraw_f : vx, zs = Pair<T>::cvt(zraw[s]);
                const float xv[2] = {xs.x, xs.y};
                const float av[2] = {(zs.x + abp[s].x) * kLog2e, (zs.y + abp[s].y) * kLog2e};
                const float m0[2] = {am[s].x, am[s].y}, l0[2] = {al_[s].x, al_[s].y}, a0[2] = {aa[s].x, aa[s].y};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    if (ai == 0) {
                        mxs[e] = av[e]; lss[e] = 1.f; acs[e] = xv[e];
                    } else {
                        const float mn = fmaxf(m0[e], av[e]);
                        const float rr = ex2(m0[e] - mn), p = ex2(av[e] - mn);
                        mxs[e] = mn; lss[e] = l0[e] * rr + p; acs[e] = fmaf(p, xv[e], a0[e] * rr);
                    }
                }
            }
            float* st = a.state + (((size_t)b * a.S + s) * 3) * GD + (size_t)g * D + 2 * tid;
            if (complete) {  // uniform across the CTA
                float e0v = acs[0] / lss[0], e1v = acs[1] / lss[1];
                const float ss = (key && a.rmsnorm)
                                     ? block_sum(pair_owner ? e0v * e0v + e1v * e1v : 0.f, scratch) : 0.f;
                if (key && a.rmsnorm) {
                    const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
                    const T* gm = static_cast<const T*>(a.gamma_kv);
                    e0v *= inv * (gm && pair_owner ? to_f<T>(gm[2 * tid]) : 1.f);
                    e1v *= inv * (gm && pair_owner ? to_f<T>(gm[2 * tid + 1]) : 1.f);
                }
                if (key && a.rho && pair_owner && 2 * tid >= D - a.rho)
                    rotate_pair(e0v, e1v, rope_cs((int64_t)aj * a.m, (2 * tid - (D - a.rho)) >> 1, a.rope_step));
                if (pair_owner) {
                    if (aj < a.max_blocks)
                        put2<T>(static_cast<T*>(key ? a.pooled_k : a.pooled_v) +
                                    (((size_t)b * a.G + g) * a.max_blocks + aj) * D + 2 * tid,
                                e0v, e1v);
                    else
                        set_status(a.status, LBCA_ERR_CAPACITY);
                }
            } else if (pair_owner) {
                *reinterpret_cast<float2*>(st) = make_float2(mxs[0], mxs[1]);
                *reinterpret_cast<float2*>(st + GD) = make_float2(lss[0], lss[1]);
                *reinterpret_cast<float2*>(st + 2 * GD) = make_float2(acs[0], acs[1]);
            }
            if (pair_owner) {  // ring slot of token t: the finalised key row, or the raw value
                T* dst = static_cast<T*>(key ? a.ring_k : a.ring_v) +
                         (((size_t)b * a.G + g) * a.R + (t % a.R)) * D + 2 * tid;
                const T* src = (key ? newk : newv) + 2 * tid;
                dst[0] = src[0];
                dst[1] = src[1];
            }
        }
    }

    const int gl = lane % LG;
    const float qscale = a.scale * kLog2e;
    float qr[R][16];
#pragma unroll
    for (int h = 0; h < R; ++h)
#pragma unroll
        for (int c = 0; c < NCH; ++c)
#pragma unroll
            for (int i = 0; i < VEC; ++i) qr[h][c * VEC + i] = qs[h * D + (c * LG + gl) * VEC + i] * qscale;

    float mx[R], ls[R], o[R][16];
#pragma unroll
    for (int h = 0; h < R; ++h) {
        mx[h] = kNegInf;
        ls[h] = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) o[h][i] = 0.f;
    }

    // ---- stream the CTA's entries through the two-stage ring ----
    bool ok = true;
    for (int st = 0; st < nst; ++st) {
        const int b0 = e0 + st * a.SE;
        const int n = min(e1, b0 + a.SE) - b0;
        T* kb = kst + (size_t)(st & 1) * a.SE * D;
        T* vb = vst + (size_t)(st & 1) * a.SE * D;
        bool okst = mbar_wait(&bars[st & 1], (uint32_t)((st >> 1) & 1));
        if (newest >= b0 && newest < b0 + n) {  // the newest row is written, not copied
            const int row = newest - b0;
            for (int i = tid; i < D / VEC; i += kThreads) {
                *reinterpret_cast<uint4*>(kb + (size_t)row * D + i * VEC) = *reinterpret_cast<const uint4*>(newk + i * VEC);
                if (!a.shared)
                    *reinterpret_cast<uint4*>(vb + (size_t)row * D + i * VEC) =
                        *reinterpret_cast<const uint4*>(newv + i * VEC);
            }
        }
        okst = __syncthreads_and(okst);
        if (!okst) {
            ok = false;
            break;
        }
        for (int eb = warp * GPW; eb < n; eb += 2 * NG) {
            const int ea = eb + lane / LG, ebb = ea + NG;
            const bool va = ea < n, vbb = ebb < n;
            const T* ka = kb + (size_t)(va ? ea : 0) * D;
            const T* kbb = kb + (size_t)(vbb ? ebb : 0) * D;
            float kfa[16], kfb[16];
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                float t0[VEC], t1[VEC];
                ld16(ka + (c * LG + gl) * VEC, t0);
                ld16(kbb + (c * LG + gl) * VEC, t1);
#pragma unroll
                for (int i = 0; i < VEC; ++i) { kfa[c * VEC + i] = t0[i]; kfb[c * VEC + i] = t1[i]; }
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
            if (!va) continue;
            const T* vra = vb + (size_t)ea * D;
            const T* vrb = vb + (size_t)(vbb ? ebb : ea) * D;
            float vfa[16], vfb[16];
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                float t0[VEC], t1[VEC];
                ld16(vra + (c * LG + gl) * VEC, t0);
                ld16(vrb + (c * LG + gl) * VEC, t1);
#pragma unroll
                for (int i = 0; i < VEC; ++i) { vfa[c * VEC + i] = t0[i]; vfb[c * VEC + i] = t1[i]; }
            }
#pragma unroll
            for (int h = 0; h < R; ++h) {
                const float sbh = vbb ? sb[h] : kNegInf;
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
        __syncthreads();  // every thread is done with this buffer
        if (tid == 0 && st + 2 < nst) issue(st + 2);
    }
    if (!ok) {
        if (tid == 0) {
            set_status(a.status, LBCA_ERR_TIMEOUT);
            mbar_wait(&bars[0], 0);  // last bounded chance for copies in flight to land
            mbar_wait(&bars[1], 0);
        }
#pragma unroll
        for (int h = 0; h < R; ++h) {
            mx[h] = kNegInf;
            ls[h] = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) o[h][i] = 0.f;
        }
    }

    griddep_launch_dependents();  // the next kernel on the stream may start its cache reads

    // ---- merge the entry groups of each warp with shuffles, then the warps ----
#pragma unroll
    for (int off = LG; off < 32; off <<= 1)
#pragma unroll
        for (int h = 0; h < R; ++h) {
            const float mo = __shfl_xor_sync(0xffffffffu, mx[h], off);
            const float lo = __shfl_xor_sync(0xffffffffu, ls[h], off);
            float M, fa, fb;
            merge_weights(mx[h], mo, M, fa, fb);
            ls[h] = ls[h] * fa + lo * fb;
#pragma unroll
            for (int i = 0; i < 16; ++i) o[h][i] = o[h][i] * fa + __shfl_xor_sync(0xffffffffu, o[h][i], off) * fb;
            mx[h] = M;
        }
    if (lane < LG) {
#pragma unroll
        for (int h = 0; h < R; ++h) {
#pragma unroll
            for (int c = 0; c < NCH; ++c)
#pragma unroll
                for (int i = 0; i < VEC; ++i)
                    wred_o[((size_t)warp * R + h) * D + (c * LG + gl) * VEC + i] = o[h][c * VEC + i];
            if (lane == 0) {
                wred_ml[(warp * R + h) * 2] = mx[h];
                wred_ml[(warp * R + h) * 2 + 1] = ls[h];
            }
        }
    }
    __syncthreads();
    // CTA partial, pushed slice by slice into the owning CTA's receive buffer
    for (int idx = tid; idx < R * D; idx += kThreads) {
        const int h = idx / D, d = idx % D;
        float M = kNegInf;
#pragma unroll
        for (int q = 0; q < kWarps; ++q) M = fmaxf(M, wred_ml[(q * R + h) * 2]);
        float Ls = 0.f, ov = 0.f;
        if (M != kNegInf) {
#pragma unroll
            for (int q = 0; q < kWarps; ++q) {
                const float f = ex2(wred_ml[(q * R + h) * 2] - M);
                ov = fmaf(wred_o[((size_t)q * R + h) * D + d], f, ov);
                Ls = fmaf(wred_ml[(q * R + h) * 2 + 1], f, Ls);
            }
        }
        const int owner = d / DS;
        float* ro = cluster.map_shared_rank(recv_o, owner);
        ro[(rank * R + h) * DS + (d - owner * DS)] = ov;
        if (d % DS == 0) {
            float* rm = cluster.map_shared_rank(recv_ml, owner);
            rm[(rank * R + h) * 2] = M;
            rm[(rank * R + h) * 2 + 1] = Ls;
        }
    }
    cluster.sync();  // every slice has landed; nothing remote is read after this

    // ---- this CTA finalises dims [rank*DS, (rank+1)*DS) of its heads: GS threads
    // per output pair, each over every GS-th rank, joined by shuffles ----
    constexpr int GS = 4;
    const int items = R * (DS / 2) * GS;
    for (int base = 0; base < items; base += kThreads) {  // every thread runs every round
        const int idx = base + tid;
        const bool act = idx < items;
        const int pr = act ? idx / GS : 0, sub = idx % GS;
        const int h = pr / (DS / 2), dl = (pr % (DS / 2)) * 2, d = rank * DS + dl;
        float M = kNegInf;
        for (int q = sub; q < CS; q += GS) M = fmaxf(M, recv_ml[(q * R + h) * 2]);
#pragma unroll
        for (int off = 1; off < GS; off <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float Ls = 0.f, o0 = 0.f, o1 = 0.f;
        if (M != kNegInf)
            for (int q = sub; q < CS; q += GS) {
                const float f = ex2(recv_ml[(q * R + h) * 2] - M);
                Ls = fmaf(recv_ml[(q * R + h) * 2 + 1], f, Ls);
                o0 = fmaf(recv_o[(q * R + h) * DS + dl], f, o0);
                o1 = fmaf(recv_o[(q * R + h) * DS + dl + 1], f, o1);
            }
#pragma unroll
        for (int off = 1; off < GS; off <<= 1) {
            Ls += __shfl_xor_sync(0xffffffffu, Ls, off);
            o0 += __shfl_xor_sync(0xffffffffu, o0, off);
            o1 += __shfl_xor_sync(0xffffffffu, o1, off);
        }
        if (!act || sub != 0) continue;
        float den = Ls;
        if (a.sink) den += (M == kNegInf) ? 1.0f : ex2(a.sink[h0 + h] * kLog2e - M);
        float v0 = den > 0.f ? o0 / den : 0.f, v1 = den > 0.f ? o1 / den : 0.f;
        if (a.shared && a.rho && d >= D - a.rho) {
            const float2 c = cs[(d - (D - a.rho)) >> 1];
            rotate_pair(v0, v1, make_float2(c.x, -c.y));
        }
        put2<T>(static_cast<T*>(a.out) + ((size_t)b * a.Hq + h0 + h) * D + d, v0, v1);
    }
}

template <typename T, int D, int R>
cudaError_t launch_step_one(const StepArgs& a, size_t smem, cudaStream_t s) {
    static bool attr_set[64] = {};  // per device
    const int dev_ = current_device();
    auto fn = decode_step_kernel<T, D, R>;
    if (dev_ < 0 || !attr_set[dev_]) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        if (dev_ >= 0) attr_set[dev_] = true;
    }
    // 16-CTA clusters are non-portable: fall back to 8 if none fits on this device
    static int max16 = -1;
    StepArgs b = a;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (b.CS > 8) {
        if (max16 < 0) {
            cfg.gridDim = dim3(16, 1, 1);
            attr[0].val.clusterDim.x = 16;
            int n = 0;
            max16 = cudaOccupancyMaxActiveClusters(&n, fn, &cfg) == cudaSuccess ? n : 0;
            cudaGetLastError();
        }
        if (max16 == 0) b.CS = 8;
    }
    cfg.gridDim = dim3(b.CS, b.Hq / R, b.B);
    attr[0].val.clusterDim.x = b.CS;
    cfg.numAttrs = b.pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, fn, b);
}
template <typename T, int D>
cudaError_t step_dispatch_r(const StepArgs& a, size_t smem, cudaStream_t s) {
    switch (a.heads_per_cta) {
        case 1: return launch_step_one<T, D, 1>(a, smem, s);
        case 2: return launch_step_one<T, D, 2>(a, smem, s);
        case 3: return launch_step_one<T, D, 3>(a, smem, s);
        case 4: return launch_step_one<T, D, 4>(a, smem, s);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t step_dispatch(const StepArgs& a, size_t smem, cudaStream_t s) {
    switch (a.D) {
        case 64: return step_dispatch_r<T, 64>(a, smem, s);
        case 128: return step_dispatch_r<T, 128>(a, smem, s);
        case 256: return step_dispatch_r<T, 256>(a, smem, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

StepPlan plan_step(int dtype, int B, int Hq, int G, int D, int m, int w, int shared, int max_ctx) {
    StepPlan p{};
    p.ok = false;
    // GQA form only: the shared form's window rows are raw entries finalised
    // by the decode kernels that read them (lbca_append then lbca_decode, or
    // the tensor-core shared-entry step)
    if ((D != 64 && D != 128 && D != 256) || w < 1 || shared) return p;
    const int r = Hq / G;
    int R = 1;
    for (int c : {4, 3, 2, 1})
        if (r % c == 0) { R = c; break; }
    const int esize = dtype == LBCA_BF16 ? 2 : 4;
    const long long groups = (long long)B * (Hq / R);
    p.heads_per_cta = R;
    // Many (sequence, head group) segments: the persistent evenly-split kernel
    // (one launch, no clusters), whose CTAs each take an equal share of all the
    // step's entries however unequal the contexts.
    const int S = shared ? 1 : 2;
    const int C = std::min(128, std::max(16, 32768 / (D * esize * S)));
    if (groups >= 96 && B <= 4096) {
        const long long mc = std::max(1, max_ctx);
        const long long P = mc > w ? (mc - w) / m : 0;
        const long long max_vis = std::min<long long>(mc, P + w + m - 1);
        p.flat = true;
        p.C = C;
        p.maxc = (int)((max_vis + C - 1) / C + 2);
        p.seg_elems = (size_t)groups;
        p.part_ml_elems = (size_t)groups * p.maxc * R * 2;
        p.part_o_elems = (size_t)groups * p.maxc * R * D;
        p.arrive_elems = 1;
        p.smem_bytes = flat_smem_bytes(dtype, B, D, R, C, shared);
        p.ok = p.smem_bytes <= 200 * 1024;
        if (p.ok) return p;
        p.flat = false;
    }
    int CS = 1;
    while (CS < 16 && CS * 2 <= D / 4 && groups * CS < 4 * 148) CS *= 2;
    p.CS = CS;
    p.SE = D >= 256 || esize == 4 ? 16 : 32;
    p.arrive_elems = (size_t)B;
    p.smem_bytes = step_layout(D, R, p.SE, esize, shared, CS).total;
    p.ok = p.smem_bytes <= 200 * 1024;
    (void)m; (void)max_ctx;
    return p;
}

static size_t a256(size_t x) { return (x + 255) / 256 * 256; }
size_t step_workspace_bytes(const StepPlan& p) {
    if (!p.flat) return a256(p.arrive_elems * 4);
    return a256(p.arrive_elems * 4) + a256(p.seg_elems * 4) + a256(p.part_ml_elems * 4) + a256(p.part_o_elems * 4);
}

cudaError_t launch_decode_step(const StepArgs& a, cudaStream_t s) {
    if (a.B == 0) return cudaSuccess;
    if (a.C > 0) return launch_decode_flat(a, s);
    const size_t smem = step_layout(a.D, a.heads_per_cta, a.SE, a.dtype == LBCA_BF16 ? 2 : 4, a.shared, a.CS).total;
    if (a.dtype == LBCA_BF16) return step_dispatch<__nv_bfloat16>(a, smem, s);
    return step_dispatch<float>(a, smem, s);
}

}  // namespace lbca
