// decode_flat.cu -- one serving step (append + decode) for large batches, as
// one persistent launch whose CTAs split the whole step's entries evenly.
//
// What is computed is lbca_append followed by lbca_decode (mSeek README, "How
// LBCA works", steps 2-5; HCA page and CSA page, "What is implemented"): the
// query of sequence b at t = L_old sees pooled entries j < P(L_old + 1) and
// raw tokens [P m, t], in one softmax with an optional sink.
//
// B200 mapping: the (sequence, head group) segments of a step hold very
// different numbers of visible entries (contexts of a batch differ by 16x), so
// a grid of one CTA group per segment leaves SMs idle behind the longest ones.
// Here the step's entries are laid end to end -- segment after segment, each
// segment its visible list -- and CTA c of the persistent grid takes the
// contiguous range [c E / N, (c + 1) E / N).  It walks the range in pieces of
// at most C entries (never across a segment), with the copies of the next two
// pieces in flight (bulk async copies into a two-buffer shared-memory ring,
// no multicast) while it computes one.  A segment that lies in one CTA's range
// is finished there; a segment cut by range boundaries leaves one partial
// (max, sum, unnormalised output) per CTA in the workspace, and the CTA that
// completes last (one atomic counter per segment, reset by that CTA) merges
// them and writes the output.  Nothing ever waits for another CTA.
//
// Every CTA reads all lengths first; the last CTA to have done so advances
// them (a grid-wide arrival counter, reset by that CTA).  The appends (one per
// sequence and kv head) are spread over the CTAs and run while their first
// copies land; nothing an append writes is read by this step's attention (the
// ring slot of t holds token t - R, a block it completes becomes visible n_win
// tokens later).  The newest raw row (token t) is built in shared memory by
// the CTA whose range ends its segment.
#include <algorithm>

#include "common.cuh"
#include "decode_common.cuh"
#include "kernels.h"

namespace lbca {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
// The step's work is split into equal shares of a sequence of entries in which
// every segment with entries is preceded by kSegCost placeholder entries: a
// CTA pays, for each segment its range starts, a query setup, a partial
// publish and shorter pieces (~7 us measured on the ragged 32-sequence batch,
// about 224 entries of piece work), so ranges that start segments are
// shortened by that much and the CTAs end together.
constexpr int kSegCost = 224;

struct FlatLayout {
    size_t args, bars, misc, lens, ecum, qs, cs, newk, newv, wred_o, wred_ml, stage, total;
};

__host__ __device__ inline size_t fal(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline FlatLayout flat_layout(int D, int R, int C, int esize, int shared, int B) {
    FlatLayout l;
    l.args = 0;                                      // a copy of the kernel arguments
    l.bars = fal(sizeof(StepArgs), 16);
    l.misc = l.bars + 16;                            // flags [4] int + block-sum scratch [kWarps]
    l.lens = l.misc + 48;
    l.ecum = fal(l.lens + (size_t)B * 4, 8);        // [B + 1] long long
    l.qs = fal(l.ecum + (size_t)(B + 1) * 8, 16);
    l.cs = l.qs + (size_t)R * D * 4;
    l.newk = fal(l.cs + (size_t)(D / 2) * 8, 16);
    l.newv = l.newk + (size_t)D * esize;
    l.wred_o = fal(l.newv + (size_t)D * esize, 16);
    l.wred_ml = l.wred_o + (size_t)kWarps * R * D * 4;
    l.stage = fal(l.wred_ml + (size_t)kWarps * R * 2 * 4, 128);
    l.total = l.stage + 2 * (size_t)C * D * esize * (shared ? 1 : 2);
    return l;
}

// Sum over the CTA (every thread must call it).
__device__ __forceinline__ float cta_sum(float v, float* scratch) {
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

// Visible entries of a sequence whose query sees L tokens (0 when the cache
// cannot hold them; the caller reports that).
__device__ __forceinline__ int vis_count(int L, int m, int w, int max_blocks, int R) {
    const int P = visible_blocks(L, m, w);
    if (P > max_blocks || L - P * m > R) return 0;
    return P + (L - P * m);
}

template <typename T, int D, int R>
__global__ void __launch_bounds__(kThreads, 3) decode_flat_kernel(const __grid_constant__ StepArgs args) {
    constexpr int VEC = Vec<T>::N;
    constexpr int LG = D / 16;        // lanes per entry
    constexpr int NCH = 16 / VEC;     // 16-byte chunks per lane
    constexpr int GPW = 32 / LG;      // entry groups per warp
    constexpr int NG = kWarps * GPW;  // entry groups per CTA
    constexpr uint32_t ROW = D * sizeof(T);

    extern __shared__ __align__(128) unsigned char smem[];
    const int C = args.C;
    const FlatLayout lay = flat_layout(D, R, C, sizeof(T), args.shared, args.B);
    // The arguments, copied once into shared memory: every later read (a table
    // entry per thread, scattered fields) is a shared-memory load instead of a
    // constant-cache miss or a serialised divergent constant read.
    static_assert(sizeof(StepArgs) % 4 == 0, "argument copy in words");
    for (int i = threadIdx.x; i < (int)(sizeof(StepArgs) / 4); i += kThreads)
        reinterpret_cast<uint32_t*>(smem + lay.args)[i] = reinterpret_cast<const uint32_t*>(&args)[i];
    __syncthreads();
    const StepArgs& a = *reinterpret_cast<const StepArgs*>(smem + lay.args);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + lay.bars);
    int* flags = reinterpret_cast<int*>(smem + lay.misc);
    float* scratch = reinterpret_cast<float*>(smem + lay.misc + 16);
    int* lens = reinterpret_cast<int*>(smem + lay.lens);
    long long* ecum = reinterpret_cast<long long*>(smem + lay.ecum);
    float* qs = reinterpret_cast<float*>(smem + lay.qs);
    float2* cs = reinterpret_cast<float2*>(smem + lay.cs);
    T* newk = reinterpret_cast<T*>(smem + lay.newk);
    T* newv = reinterpret_cast<T*>(smem + lay.newv);
    float* wred_o = reinterpret_cast<float*>(smem + lay.wred_o);
    float* wred_ml = reinterpret_cast<float*>(smem + lay.wred_ml);
    T* kst = reinterpret_cast<T*>(smem + lay.stage);           // [2][C][D]
    T* vst = a.shared ? kst : kst + 2 * (size_t)C * D;          // [2][C][D]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = a.Hq / a.G, HG = a.Hq / R, GD = a.G * D;
    const int B = a.B;

    // ---- every length, once; the last CTA to have read them advances them ----
    for (int b = tid; b < B; b += kThreads) lens[b] = a.seq_lens[b];
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_barrier_init();
    }
    __syncthreads();
    // arrival ticket: taken once the step's inputs may be read (below), looked at
    // only at the end (its latency hides behind the work)
    unsigned int ticket = 0u;
    // exclusive prefix of the step's entries per sequence (HG segments of kSegCost
    // placeholders then nvis entries each; none for a sequence without entries)
    {
        const int per = (B + kThreads - 1) / kThreads;
        const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
        long long sum = 0;
        for (int b = b0; b < b1; ++b) {
            const int nv = vis_count(lens[b] + 1, a.m, a.w, a.max_blocks, a.R);
            if (nv == 0 && blockIdx.x == 0) set_status(a.status, LBCA_ERR_CAPACITY);
            sum += nv ? (long long)HG * (nv + kSegCost) : 0;
        }
        long long incl = sum;  // inclusive scan over the warp
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        long long* wsum = reinterpret_cast<long long*>(wred_o);  // scratch before any use of wred_o
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        long long base = 0;
        for (int q = 0; q < warp; ++q) base += wsum[q];
        long long run = base + incl - sum;
        for (int b = b0; b < b1; ++b) {
            ecum[b] = run;
            const int nv = vis_count(lens[b] + 1, a.m, a.w, a.max_blocks, a.R);
            run += nv ? (long long)HG * (nv + kSegCost) : 0;
        }
        if (tid == kThreads - 1) ecum[B] = base + incl;
    }
    __syncthreads();

    // ---- this CTA's range of the step's entries ----
    const long long E = ecum[B];
    // active CTAs: each takes at least C positions, so a segment of n entries has
    // at most n / C + 2 contributors
    const long long NA = std::max<long long>(1, std::min<long long>((long long)gridDim.x, E / C));
    const int cta = blockIdx.x;
    const long long e_lo = cta < NA ? cta * E / NA : 0;
    const long long e_hi = cta < NA ? (cta + 1) * E / NA : 0;
    auto ctaof = [&](long long e) { return (int)(((e + 1) * NA - 1) / E); };
    // sequence of entry e: the last b with ecum[b] <= e
    auto seq_of = [&](long long e) {
        int lo = 0, hi = B - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (ecum[mid] <= e) lo = mid; else hi = mid - 1;
        }
        return lo;
    };

    // ---- piece cursor: (sequence, head group, entry within the segment) of a
    // position, advanced piece by piece without searching; placeholders are
    // skipped (a cursor past e_hi ends the walk) ----
    struct Cursor {
        long long e;
        int b, hg, j, nv, P;
    };
    // position of the first entry of segment (b, hg) whose sequence has nv entries
    auto seg_first = [&](int b, int hg, int nv) {
        return ecum[b] + (long long)hg * (nv + kSegCost) + kSegCost;
    };
    auto cursor_at = [&](long long e0) {
        Cursor c{e0, 0, 0, 0, 1, 0};
        if (e0 >= e_hi) return c;
        c.b = seq_of(e0);
        const int L = lens[c.b] + 1;
        c.nv = vis_count(L, a.m, a.w, a.max_blocks, a.R);
        c.P = visible_blocks(L, a.m, a.w);
        const int loc = (int)(e0 - ecum[c.b]);
        c.hg = loc / (c.nv + kSegCost);
        c.j = loc - c.hg * (c.nv + kSegCost) - kSegCost;
        if (c.j < 0) {  // a placeholder: the segment's first entry
            c.e -= c.j;
            c.j = 0;
        }
        return c;
    };
    auto piece_len = [&](const Cursor& c) { return (int)std::min<long long>(std::min(c.nv - c.j, C), e_hi - c.e); };
    auto advance = [&](Cursor& c, int n) {
        c.e += n;
        c.j += n;
        if (c.j == c.nv && c.e < e_hi) {  // next segment: next head group, or the next sequence with entries
            c.j = 0;
            c.e += kSegCost;
            if (++c.hg == HG) {
                c.hg = 0;
                do {
                    ++c.b;
                    const int L = lens[c.b] + 1;
                    c.nv = vis_count(L, a.m, a.w, a.max_blocks, a.R);
                    c.P = visible_blocks(L, a.m, a.w);
                } while (c.nv == 0);
            }
        }
    };

    // ---- copies of the piece at cursor c into buffer buf (thread 0); returns its size ----
    auto issue = [&](const Cursor& c, int buf) -> int {
        const int b = c.b, j = c.j, P = c.P, s0 = P * a.m;
        const int n = piece_len(c);
        const int g = c.hg * R / r;
        const int c1 = min(j + n, c.nv - 1);  // rows [j, c1) come from memory; the newest is built
        const uint32_t rows = c1 > j ? (uint32_t)(c1 - j) : 0u;
        T* kd = kst + (size_t)buf * C * D;
        T* vd = vst + (size_t)buf * C * D;
        mbar_arrive_expect_tx(&bars[buf], rows * ROW * (a.shared ? 1u : 2u));
        const size_t pool_head = ((size_t)b * a.G + g) * a.max_blocks;
        const size_t ring_head = ((size_t)b * a.G + g) * a.R;
        int idx = j, row = 0;
        if (idx < c1 && idx < P) {
            const int cnt = min(c1, P) - idx;
            bulk_g2s(kd, static_cast<const T*>(a.pooled_k) + (pool_head + checked_rows(idx, cnt, a.max_blocks, a.status)) * D, cnt * ROW, &bars[buf]);
            if (!a.shared)
                bulk_g2s(vd, static_cast<const T*>(a.pooled_v) + (pool_head + checked_rows(idx, cnt, a.max_blocks, a.status)) * D, cnt * ROW, &bars[buf]);
            idx += cnt;
            row += cnt;
        }
        while (idx < c1) {
            const int slot = (s0 + (idx - P)) % a.R;
            const int cnt = min(c1 - idx, a.R - slot);
            bulk_g2s(kd + (size_t)row * D, static_cast<const T*>(a.ring_k) + (ring_head + checked_rows(slot, cnt, a.R, a.status)) * D, cnt * ROW,
                     &bars[buf]);
            if (!a.shared)
                bulk_g2s(vd + (size_t)row * D, static_cast<const T*>(a.ring_v) + (ring_head + checked_rows(slot, cnt, a.R, a.status)) * D,
                         cnt * ROW, &bars[buf]);
            idx += cnt;
            row += cnt;
        }
        return n;
    };
    Cursor iss = cursor_at(e_lo);  // issue cursor (thread 0)
    // the first two pieces go out right after this CTA's first append has issued its
    // few loads (ahead of the copies in the memory queues)
    bool issued = false;
    auto issue_first = [&]() {
        if (tid == 0)
            for (int buf = 0; buf < 2 && iss.e < e_hi; ++buf) advance(iss, issue(iss, buf));
        issued = true;
    };

    const bool pair_owner = tid < D / 2;

    // Everything above reads only this cache.  Launched with programmatic
    // dependence on the preceding kernel, the first pieces' copies go out now,
    // while that kernel drains; otherwise after the first append's few loads
    // (ahead of the copies in the memory queues).  The step's own inputs (the
    // new tokens, the queries) and the workspace are touched only after the wait.
    if (a.pdl) issue_first();
    griddep_wait();
    if (tid == 0) ticket = atomicAdd(a.arrive, 1u);

    // ---- appends of (sequence, kv head) pairs c, c + N, ... while the copies land ----
    const int kp = pair_owner && a.rho && 2 * tid >= D - a.rho ? (2 * tid - (D - a.rho)) >> 1 : -1;  // RoPE pair
    for (int pidx = cta; pidx < B * a.G; pidx += gridDim.x) {
        const int b = pidx / a.G, g = pidx % a.G;
        const int t = lens[b];
        const int ai = t % a.m, aj = t / a.m;
        const bool complete = ai == a.m - 1;
        const size_t tok = (size_t)b * GD + (size_t)g * D + 2 * tid;
        // every load first: the token, its pooling logits, the B_pos rows, the open block's state
        float2 xr[2] = {}, zr[2] = {}, bp[2] = {}, sm[2] = {}, sl[2] = {}, sa[2] = {};
        if (pair_owner) {
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                if (s >= a.S) break;
                xr[s] = get2(static_cast<const T*>(s == 0 ? a.k : a.v) + tok);
                zr[s] = get2(static_cast<const T*>(s == 0 ? a.zk : a.zv) + tok);
                bp[s] = get2(static_cast<const T*>(s == 0 ? a.bpk : a.bpv) + (size_t)ai * GD + (size_t)g * D + 2 * tid);
                const float* st = a.state + (((size_t)b * a.S + s) * 3) * GD + (size_t)g * D + 2 * tid;
                sm[s] = *reinterpret_cast<const float2*>(st);
                sl[s] = *reinterpret_cast<const float2*>(st + GD);
                sa[s] = *reinterpret_cast<const float2*>(st + 2 * GD);
            }
        }
        if (!issued) issue_first();
        // the raw token's finalised key (RMSNorm, RoPE at t) for the ring
        float2 kf = xr[0];
        const float ssk = a.rmsnorm ? cta_sum(pair_owner ? kf.x * kf.x + kf.y * kf.y : 0.f, scratch) : 0.f;
        if (pair_owner) {
            if (a.rmsnorm) {
                const float inv = 1.0f / sqrtf(ssk / (float)D + a.eps);
                const T* gm = static_cast<const T*>(a.gamma_kv);
                kf.x *= inv * (gm ? to_f<T>(gm[2 * tid]) : 1.f);
                kf.y *= inv * (gm ? to_f<T>(gm[2 * tid + 1]) : 1.f);
            }
            if (kp >= 0) rotate_pair(kf.x, kf.y, rope_cs_turns((int64_t)t, a.rope_f[kp]));
        }
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            if (s >= a.S) break;
            const bool key = s == 0;
            float mxs[2] = {0.f, 0.f}, lss[2] = {1.f, 1.f}, acs[2] = {0.f, 0.f};
            if (pair_owner) {
                const float xv[2] = {xr[s].x, xr[s].y};
                const float av[2] = {(zr[s].x + bp[s].x) * kLog2e, (zr[s].y + bp[s].y) * kLog2e};
                const float m0[2] = {sm[s].x, sm[s].y}, l0[2] = {sl[s].x, sl[s].y}, a0[2] = {sa[s].x, sa[s].y};
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
            if (complete) {  // uniform across the CTA
                float e0v = acs[0] / lss[0], e1v = acs[1] / lss[1];
                const float ss = (key && a.rmsnorm) ? cta_sum(pair_owner ? e0v * e0v + e1v * e1v : 0.f, scratch)
                                                    : 0.f;
                if (key && a.rmsnorm) {
                    const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
                    const T* gm = static_cast<const T*>(a.gamma_kv);
                    e0v *= inv * (gm && pair_owner ? to_f<T>(gm[2 * tid]) : 1.f);
                    e1v *= inv * (gm && pair_owner ? to_f<T>(gm[2 * tid + 1]) : 1.f);
                }
                if (key && kp >= 0) rotate_pair(e0v, e1v, rope_cs_turns((int64_t)aj * a.m, a.rope_f[kp]));
                if (pair_owner) {
                    if (aj < a.max_blocks)
                        put2<T>(static_cast<T*>(key ? a.pooled_k : a.pooled_v) +
                                    (((size_t)b * a.G + g) * a.max_blocks + aj) * D + 2 * tid,
                                e0v, e1v);
                    else
                        set_status(a.status, LBCA_ERR_CAPACITY);
                }
            } else if (pair_owner) {
                float* st = a.state + (((size_t)b * a.S + s) * 3) * GD + (size_t)g * D + 2 * tid;
                *reinterpret_cast<float2*>(st) = make_float2(mxs[0], mxs[1]);
                *reinterpret_cast<float2*>(st + GD) = make_float2(lss[0], lss[1]);
                *reinterpret_cast<float2*>(st + 2 * GD) = make_float2(acs[0], acs[1]);
            }
            if (pair_owner) {  // ring slot of token t: the finalised key, or the raw value
                const float2 rv = key ? kf : xr[s];
                put2<T>(static_cast<T*>(key ? a.ring_k : a.ring_v) + (((size_t)b * a.G + g) * a.R + (t % a.R)) * D +
                            2 * tid,
                        rv.x, rv.y);
            }
        }
    }

    if (!issued) issue_first();

    // ---- sequences whose cache could not hold the step: zero outputs ----
    for (int seg = cta; seg < B * HG; seg += gridDim.x) {
        const int b = seg / HG;
        if (vis_count(lens[b] + 1, a.m, a.w, a.max_blocks, a.R) > 0) continue;
        for (int idx = tid; idx < R * D / 2; idx += kThreads)
            put2<T>(static_cast<T*>(a.out) + ((size_t)b * a.Hq + (seg % HG) * R) * D + 2 * idx, 0.f, 0.f);
    }

    // ---- the range, piece by piece ----
    const int gl = lane % LG;
    float qr[R][16];
    float mx[R], ls[R], o[R][16];
    int seg_cur = -1, b_cur = 0, hg_cur = 0, nv_cur = 1, t_cur = 0;
    bool ok = true;
    int k = 0;

    // Output pair (d, d + 1) of head h of segment (b, hg) from its merged
    // (max, sum, unnormalised output): sink, normalisation, -t turn (shared form).
    auto emit = [&](int b, int hg, int h, int d, float M, float Ls, float o0, float o1) {
        const int h0 = hg * R;
        float den = Ls;
        if (a.sink) den += (M == kNegInf) ? 1.0f : ex2(a.sink[h0 + h] * kLog2e - M);
        float v0 = den > 0.f ? o0 / den : 0.f, v1 = den > 0.f ? o1 / den : 0.f;
        if (a.shared && a.rho && d >= D - a.rho) {
            const float2 c = rope_cs_turns((int64_t)lens[b], a.rope_f[(d - (D - a.rho)) >> 1]);
            rotate_pair(v0, v1, make_float2(c.x, -c.y));
        }
        put2<T>(static_cast<T*>(a.out) + ((size_t)b * a.Hq + h0 + h) * D + d, v0, v1);
    };
    // Merge of every contributor's partial of segment seg (by its last contributor).
    auto merge = [&](int seg, int ncon) {
        const size_t slot0 = (size_t)seg * a.maxc;
        for (int idx = tid; idx < R * D / 2; idx += kThreads) {
            const int h = idx / (D / 2), d = (idx % (D / 2)) * 2;
            // every partial's (max, sum) and output pair in one batch of loads, 8 at a time
            float M = kNegInf, Ls = 0.f, o0 = 0.f, o1 = 0.f;
            for (int q0 = 0; q0 < ncon; q0 += 8) {
                float2 ml[8], po[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const size_t sl = slot0 + min(q0 + u, ncon - 1);
                    ml[u] = __ldcg(reinterpret_cast<const float2*>(a.part_ml + (sl * R + h) * 2));
                    po[u] = __ldcg(reinterpret_cast<const float2*>(a.part_o + (sl * R + h) * D + d));
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (q0 + u >= ncon || ml[u].x == kNegInf) continue;
                    float Mn, fa, fb;
                    merge_weights(M, ml[u].x, Mn, fa, fb);
                    Ls = Ls * fa + ml[u].y * fb;
                    o0 = o0 * fa + po[u].x * fb;
                    o1 = o1 * fa + po[u].y * fb;
                    M = Mn;
                }
            }
            emit(seg / HG, seg % HG, h, d, M, Ls, o0, o1);
        }
        if (tid == 0) a.seg_count[seg] = 0u;
    };

    // End of the CTA's share of segment (b_cur, hg_cur): CTA partial, then the
    // output (sole contributor) or the workspace partial (and, for the last
    // contributor, the merge of all of them).
    auto finish = [&]() {
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
                for (int i = 0; i < 16; ++i)
                    o[h][i] = o[h][i] * fa + __shfl_xor_sync(0xffffffffu, o[h][i], off) * fb;
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
        const int seg = seg_cur;
        const long long es = seg_first(b_cur, hg_cur, nv_cur), ee = es + nv_cur;
        const int c_first = ctaof(es), ncon = ctaof(ee - 1) - c_first + 1;
        if (ncon > a.maxc) {  // more contributors than the workspace was sized for (max_ctx too small)
            if (tid == 0) set_status(a.status, LBCA_ERR_CAPACITY);
            __syncthreads();
            return;
        }
        const int h0 = hg_cur * R;
        if (ncon == 1) {
            for (int idx = tid; idx < R * D / 2; idx += kThreads) {
                const int h = idx / (D / 2), d = (idx % (D / 2)) * 2;
                float M = kNegInf;
#pragma unroll
                for (int q = 0; q < kWarps; ++q) M = fmaxf(M, wred_ml[(q * R + h) * 2]);
                float Ls = 0.f, o0 = 0.f, o1 = 0.f;
                if (M != kNegInf) {
#pragma unroll
                    for (int q = 0; q < kWarps; ++q) {
                        const float f = ex2(wred_ml[(q * R + h) * 2] - M);
                        Ls = fmaf(wred_ml[(q * R + h) * 2 + 1], f, Ls);
                        o0 = fmaf(wred_o[((size_t)q * R + h) * D + d], f, o0);
                        o1 = fmaf(wred_o[((size_t)q * R + h) * D + d + 1], f, o1);
                    }
                }
                emit(b_cur, hg_cur, h, d, M, Ls, o0, o1);
            }
        } else {
            const size_t slot0 = (size_t)seg * a.maxc;
            const int slot = cta - c_first;
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
                        Ls = fmaf(wred_ml[(q * R + h) * 2 + 1], f, Ls);
                        ov = fmaf(wred_o[((size_t)q * R + h) * D + d], f, ov);
                    }
                }
                a.part_o[((slot0 + slot) * R + h) * D + d] = ov;
                if (d == 0) {
                    a.part_ml[((slot0 + slot) * R + h) * 2] = M;
                    a.part_ml[((slot0 + slot) * R + h) * 2 + 1] = Ls;
                }
            }
            __syncthreads();  // every partial of this CTA is written ...
            if (tid == 0) {   // ... and published (a fence cumulative over the CTA barrier), then counted
                __threadfence();
                const bool last = atomicAdd(&a.seg_count[seg], 1u) == (uint32_t)(ncon - 1);
                if (last) __threadfence();  // the other contributors' partials are visible from here
                flags[1] = last;
            }
            __syncthreads();
            if (flags[1]) merge(seg, ncon);  // the last contributor merges every partial
        }
        __syncthreads();  // wred and cs are reused
    };

    Cursor cur = cursor_at(e_lo);
    while (cur.e < e_hi) {
        const int b = cur.b, nv = cur.nv, hg = cur.hg, j = cur.j;
        const int n = piece_len(cur);
        const int seg = b * HG + hg;
        if (seg != seg_cur) {
            if (seg_cur >= 0) finish();
            // ---- a new segment: its query heads at t, and its newest row if this range ends it ----
            seg_cur = seg; b_cur = b; hg_cur = hg; nv_cur = nv; t_cur = lens[b];
            const int h0 = hg * R, g = h0 / r;
            for (int kk = tid; kk < a.rho / 2; kk += kThreads) cs[kk] = rope_cs_turns((int64_t)t_cur, a.rope_f[kk]);
            for (int idx = tid; idx < R * D / VEC; idx += kThreads) {
                const int h = idx / (D / VEC), c = idx % (D / VEC);
                float v[VEC];
                ld16(static_cast<const T*>(a.q) + ((size_t)b * a.Hq + h0 + h) * D + c * VEC, v);
#pragma unroll
                for (int i = 0; i < VEC; ++i) qs[h * D + c * VEC + i] = v[i];
            }
            const bool ends_here = seg_first(b, hg, nv) + nv - 1 < e_hi;  // uniform
            float2 kx = make_float2(0.f, 0.f), vx = kx;
            if (ends_here && pair_owner) {
                const size_t tok = (size_t)b * GD + (size_t)g * D + 2 * tid;
                kx = get2(static_cast<const T*>(a.k) + tok);
                if (!a.shared) vx = get2(static_cast<const T*>(a.v) + tok);
            }
            __syncthreads();  // cs, qs
            if (ends_here) {
                const float ss = a.rmsnorm ? cta_sum(pair_owner ? kx.x * kx.x + kx.y * kx.y : 0.f, scratch) : 0.f;
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
                const int h = idx / (a.rho / 2), kk = idx % (a.rho / 2);
                const int d = D - a.rho + 2 * kk;
                rotate_pair(qs[h * D + d], qs[h * D + d + 1], cs[kk]);
            }
            __syncthreads();
            const float qscale = a.scale * kLog2e;
#pragma unroll
            for (int h = 0; h < R; ++h)
#pragma unroll
                for (int c = 0; c < NCH; ++c)
#pragma unroll
                    for (int i = 0; i < VEC; ++i) qr[h][c * VEC + i] = qs[h * D + (c * LG + gl) * VEC + i] * qscale;
#pragma unroll
            for (int h = 0; h < R; ++h) {
                mx[h] = kNegInf;
                ls[h] = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) o[h][i] = 0.f;
            }
        }

        // ---- this piece's rows: landed copies, plus the newest row if it is here ----
        const int buf = k & 1;
        T* kb = kst + (size_t)buf * C * D;
        T* vb = vst + (size_t)buf * C * D;
        bool okp = ok && mbar_wait(&bars[buf], (uint32_t)((k >> 1) & 1));
        const int newest = nv - 1;
        if (newest >= j && newest < j + n) {
            const int row = newest - j;
            for (int i = tid; i < D / VEC; i += kThreads) {
                *reinterpret_cast<uint4*>(kb + (size_t)row * D + i * VEC) = *reinterpret_cast<const uint4*>(newk + i * VEC);
                if (!a.shared)
                    *reinterpret_cast<uint4*>(vb + (size_t)row * D + i * VEC) =
                        *reinterpret_cast<const uint4*>(newv + i * VEC);
            }
        }
        okp = __syncthreads_and(okp);
        if (!okp && ok) {
            ok = false;
            if (tid == 0) set_status(a.status, LBCA_ERR_TIMEOUT);
        }
        if (ok) {
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
        }
        __syncthreads();  // every thread is done with this buffer
        if (tid == 0 && ok && iss.e < e_hi) advance(iss, issue(iss, buf));
        advance(cur, n);
        ++k;
    }
    griddep_launch_dependents();  // the next kernel on the stream may start its cache reads
    if (seg_cur >= 0) finish();
    // ---- the last CTA to have read the lengths advances them ----
    if (tid == 0) flags[0] = ticket == gridDim.x - 1;
    __syncthreads();
    if (flags[0]) {
        for (int b = tid; b < B; b += kThreads) a.seq_lens[b] = lens[b] + 1;
        if (tid == 0) *a.arrive = 0u;
    }
    if (!ok && tid == 0) {  // last bounded chance for copies in flight to land
        mbar_wait(&bars[0], (uint32_t)((k >> 1) & 1));
        mbar_wait(&bars[1], (uint32_t)((k >> 1) & 1));
    }
}

template <typename T, int D, int R>
cudaError_t flat_attr() {
    static bool attr_set[64] = {};  // per device
    const int dev_ = current_device();
    if (dev_ < 0 || !attr_set[dev_]) {
        cudaError_t e = cudaFuncSetAttribute(decode_flat_kernel<T, D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             200 * 1024);
        if (e != cudaSuccess) return e;
        if (dev_ >= 0) attr_set[dev_] = true;
    }
    return cudaSuccess;
}
template <typename T, int D, int R>
cudaError_t launch_flat_one(const StepArgs& a, size_t smem, cudaStream_t s) {
    cudaError_t e = flat_attr<T, D, R>();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(a.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_flat_kernel<T, D, R>, a);
}
// Persistent grid: every SM filled with as many CTAs as fit (cached per device and shape).
template <typename T, int D, int R>
cudaError_t grid_one(int* grid, size_t smem) {
    static int cached = 0, cached_dev = -1;
    static size_t cached_smem = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (cached > 0 && cached_dev == dev && cached_smem == smem) {
        *grid = cached;
        return cudaSuccess;
    }
    if ((e = flat_attr<T, D, R>()) != cudaSuccess) return e;
    int per_sm = 0, sms = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_flat_kernel<T, D, R>, kThreads, smem)) !=
        cudaSuccess)
        return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached = std::max(1, per_sm) * std::max(1, sms);
    cached_dev = dev;
    cached_smem = smem;
    *grid = cached;
    return cudaSuccess;
}
template <typename T, int D>
cudaError_t grid_r(int* grid, int R, size_t smem) {
    switch (R) {
        case 1: return grid_one<T, D, 1>(grid, smem);
        case 2: return grid_one<T, D, 2>(grid, smem);
        case 3: return grid_one<T, D, 3>(grid, smem);
        case 4: return grid_one<T, D, 4>(grid, smem);
        default: return cudaErrorInvalidValue;
    }
}
template <typename T>
cudaError_t grid_d(int* grid, int D, int R, size_t smem) {
    switch (D) {
        case 64: return grid_r<T, 64>(grid, R, smem);
        case 128: return grid_r<T, 128>(grid, R, smem);
        case 256: return grid_r<T, 256>(grid, R, smem);
        default: return cudaErrorInvalidValue;
    }
}
template <typename T, int D>
cudaError_t flat_dispatch_r(const StepArgs& a, size_t smem, cudaStream_t s) {
    switch (a.heads_per_cta) {
        case 1: return launch_flat_one<T, D, 1>(a, smem, s);
        case 2: return launch_flat_one<T, D, 2>(a, smem, s);
        case 3: return launch_flat_one<T, D, 3>(a, smem, s);
        case 4: return launch_flat_one<T, D, 4>(a, smem, s);
        default: return cudaErrorInvalidValue;
    }
}
template <typename T>
cudaError_t flat_dispatch(const StepArgs& a, size_t smem, cudaStream_t s) {
    switch (a.D) {
        case 64: return flat_dispatch_r<T, 64>(a, smem, s);
        case 128: return flat_dispatch_r<T, 128>(a, smem, s);
        case 256: return flat_dispatch_r<T, 256>(a, smem, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

size_t flat_smem_bytes(int dtype, int B, int D, int R, int C, int shared) {
    return flat_layout(D, R, C, dtype == LBCA_BF16 ? 2 : 4, shared, B).total;
}

cudaError_t flat_grid(int* grid, int dtype, int D, int R, size_t smem) {
    return dtype == LBCA_BF16 ? grid_d<__nv_bfloat16>(grid, D, R, smem) : grid_d<float>(grid, D, R, smem);
}

cudaError_t launch_decode_flat(const StepArgs& a, cudaStream_t s) {
    if (a.B == 0) return cudaSuccess;
    const size_t smem = flat_smem_bytes(a.dtype, a.B, a.D, a.heads_per_cta, a.C, a.shared);
    if (a.dtype == LBCA_BF16) return flat_dispatch<__nv_bfloat16>(a, smem, s);
    return flat_dispatch<float>(a, smem, s);
}

}  // namespace lbca
