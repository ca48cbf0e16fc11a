// decode_mqa_tc.cu -- tensor-core decode for the shared-entry (MQA) form.
//
// One query per sequence at position t = L - 1 attends, in one softmax, to the
// visible pooled entries j < P(L) and the raw tokens s in [P(L) m, t], plus an
// optional sink logit that only enters the denominator; keys and values are
// the same finalised entries E, and the output's rotated dims turn back by -t
// (HCA page, "What is implemented": MQA shared KV, RMSNorm on queries and
// entries, partial RoPE, attention sink; CSA page, "What is implemented":
// Eqs 18-19, Eq 27 and the -i output rotation; mSeek README, "How LBCA
// works", step 4 for the visible set).
//
// In this form all NH = Hq / G query heads of a kv head read the same entries,
// so one entry row of D bf16 values serves 4 NH flops per byte -- 128 flop/B
// at NH = 64, too many for CUDA cores to keep up with HBM.  Both products run
// on tcgen05 tensor cores with the entries as the M = 128 operand:
//
//   S^T = E . Q^T    M = 128 entry rows, N = NH heads, K = D     (A, B K-major)
//   O^T = E^T . P^T  M = 128 dims (D / 128 tiles), N = NH, K = entries
//                    (A = the same E tile read MN-major, B = P^T MN-major)
//
// so each entry tile crosses HBM once and shared memory feeds both MMAs.  The
// MMAs take fp16 operands: the bf16 entries are widened to fp16 in shared
// memory (exact for every bf16 value of magnitude 2^-14 .. 65504; RMSNorm
// keeps entries and queries far inside that), and Q and P are rounded to
// fp16, whose 11-bit significand keeps the weights 8x closer than bf16 would.
// An element beyond the fp16 range sets d_status to LBCA_ERR_UNSUPPORTED.
//
// B200 mapping: grid (CS, G, B) with cluster (CS, 1, 1).  The CS CTAs of a
// cluster split one (sequence, kv head)'s visible list into CS chunks of at
// most 128 entries.  A CTA copies its chunk (pooled rows, then ring rows) into
// 128-byte-swizzled shared memory with 16-byte cp.async, prepares the NH
// queries meanwhile (RMSNorm, RoPE at t, fp16, swizzled), issues the S^T MMAs
// (one thread), takes the per-head max and sum over its entries with
// transposing warp butterflies, writes P^T (fp16) and issues the O^T MMAs.
// The partials are merged inside the cluster through distributed shared
// memory: after one cluster barrier every CTA reads all CTAs' (max, sum) per
// head, scales its O^T by 2^(m - M) / denominator (the sink joins the
// denominator), and pushes slice d / (D / CS) of it to the CTA that owns those
// dims; after a second barrier each CTA sums its slice, turns the rotated dims
// back by -t and writes the output.  No workspace, no second launch.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace cg = cooperative_groups;

namespace lbca {
namespace {

constexpr int kThreads = 256;
constexpr int NH = 64;          // query heads per kv head (N of both MMAs)
constexpr int TE = 128;         // entry rows per CTA tile (M of S^T)
constexpr uint64_t kWaitNs = 200ull * 1000 * 1000;

template <int D>
struct MqaLayout {
    static constexpr uint32_t EREG = TE * 128;               // one 64-dim column region of E
    static constexpr uint32_t QREG = NH * 128;               // one 64-dim column region of Q
    static constexpr uint32_t OFF_E = 0;
    static constexpr uint32_t OFF_Q = OFF_E + (D / 64) * EREG;
    static constexpr uint32_t OFF_P = OFF_Q + (D / 64) * QREG;
    static constexpr uint32_t OFF_CS = OFF_P + TE * NH * 2;  // [D/2] float2 cos/sin at t
    static constexpr uint32_t OFF_RED = OFF_CS + (D / 2) * 8;  // [2][4][NH] warp partials
    static constexpr uint32_t OFF_MH = OFF_RED + 2 * 4 * NH * 4;  // [NH] CTA max
    static constexpr uint32_t OFF_ML = OFF_MH + NH * 4;            // [2][NH] published (max, sum)
    static constexpr uint32_t OFF_F = OFF_ML + 2 * NH * 4;         // [NH] merge factor
    static constexpr uint32_t OFF_BAR = OFF_F + NH * 4;            // 2 mbarriers, TMEM base, flag
    static constexpr uint32_t TOTAL = OFF_BAR + 64;
    static constexpr uint32_t SMEM = TOTAL + 1024;                 // slack for 1024-byte alignment
    // the merge's receive buffer [CS][NH/4][D/CS][4] f32 = NH * D * 4 bytes aliases E and Q
    static_assert((uint32_t)NH * D * 4 <= OFF_P, "receive buffer must fit in the E and Q regions");
    static constexpr uint32_t TMEM_COLS = (NH + (D / 128) * NH) <= 256 ? 256 : 512;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Butterfly over the 32 lanes of a warp that leaves lane l holding the
// reduction over all lanes of v[l]: each step trades half of the remaining
// values with the partner lane, 31 shuffles in all.
template <bool kMax>
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float send = up ? v[i] : v[i + o];
            const float keep = up ? v[i + o] : v[i];
            const float got = __shfl_xor_sync(0xffffffffu, send, o);
            v[i] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
    return v[0];
}

// kind::f16 instruction descriptor with both operands MN-major (fp16 in, f32 out).
__host__ __device__ constexpr uint32_t idesc_f16_f32_mn_mn(int M, int N) {
    return (1u << 4) | (1u << 15) | (1u << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

constexpr float kF16Max = 65504.f;

// Two bf16 -> two fp16 (exact inside the fp16 range); flags values beyond it.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, bool& ovf) {
    const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xffff0000u);
    ovf |= fabsf(lo) > kF16Max || fabsf(hi) > kF16Max;
    return pack_f16x2(lo, hi);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) decode_mqa_tc_kernel(const DecodeArgs a) {
    using Lay = MqaLayout<D>;
    constexpr int CPL = D / 256;  // 16-byte query chunks per lane per head
    static_assert(D % 256 == 0 && D <= 512, "D must be 256 or 512");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
    uint32_t* tmem_sh = reinterpret_cast<uint32_t*>(smem + Lay::OFF_BAR + 16);
    float2* cs = reinterpret_cast<float2*>(smem + Lay::OFF_CS);
    float* red = reinterpret_cast<float*>(smem + Lay::OFF_RED);
    float* mh = reinterpret_cast<float*>(smem + Lay::OFF_MH);
    float* ml = reinterpret_cast<float*>(smem + Lay::OFF_ML);
    float* fh = reinterpret_cast<float*>(smem + Lay::OFF_F);
    float* recv = reinterpret_cast<float*>(smem + Lay::OFF_E);

    cg::cluster_group cluster = cg::this_cluster();
    const int CS = a.tc_cs;
    const int rank = (int)blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int SW = D / CS;  // output dims owned by each CTA of the cluster

    // ---- visible set of this sequence (block-aligned partition) and this CTA's chunk ----
    const int L = a.seq_lens[b];
    const int t = L - 1;
    const int P = visible_blocks(L, a.m, a.w);
    const int s0 = P * a.m;
    int n_vis = L > 0 ? P + (L - s0) : 0;
    if (P > a.max_blocks || L - s0 > a.R || n_vis > TE * CS) {  // cache or split grid cannot hold it
        if (rank == 0 && g == 0 && tid == 0) set_status(a.status, LBCA_ERR_CAPACITY);
        n_vis = 0;
    }
    const int chunk = (n_vis + CS - 1) / CS;
    const int e0 = rank * chunk;
    const int n = max(0, min(n_vis, e0 + chunk) - e0);
    const int n16 = (n + 15) & ~15;

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_barrier_init();
    }
    __syncwarp();
    if (warp == 0) tmem_alloc(tmem_sh, Lay::TMEM_COLS);

    // ---- stage the chunk's entry rows (bf16), 128-byte swizzled; rows [n, n16) zero ----
    const uint32_t sE = smem_addr(smem + Lay::OFF_E);
    {
        const size_t pool_head = ((size_t)b * a.G + g) * a.max_blocks;
        const size_t ring_head = ((size_t)b * a.G + g) * a.R;
        const __nv_bfloat16* pk = static_cast<const __nv_bfloat16*>(a.pooled_k);
        const __nv_bfloat16* rk = static_cast<const __nv_bfloat16*>(a.ring_k);
        constexpr int CPR = D / 8;  // 16-byte chunks per row
        for (int c = tid; c < n16 * CPR; c += kThreads) {
            const int row = c / CPR, ch = c % CPR;
            const uint32_t dst = sE + (uint32_t)(ch >> 3) * Lay::EREG + (uint32_t)(row >> 3) * 1024u +
                                 (uint32_t)(row & 7) * 128u + ((uint32_t)((ch & 7) ^ (row & 7)) << 4);
            const void* src = a.q;  // any valid address for the zero-filled rows
            uint32_t bytes = 0;
            if (row < n) {
                const int idx = e0 + row;
                src = idx < P ? pk + (pool_head + idx) * D + ch * 8
                              : rk + (ring_head + (s0 + (idx - P)) % a.R) * D + ch * 8;
                bytes = 16;
            }
            cp_async16(dst, src, bytes);
        }
    }

    // ---- cos/sin at t, then the NH queries: RMSNorm, RoPE, fp16, swizzled (K-major) ----
    for (int k = tid; k < a.rho / 2; k += kThreads) cs[k] = rope_cs((int64_t)t, k, a.rope_step);
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_sh;
    bool ovf = false;
    {
        const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q) + ((size_t)b * a.Hq + (size_t)g * NH) * D;
        const __nv_bfloat16* gm = static_cast<const __nv_bfloat16*>(a.gamma_q);
        float gam[CPL][8];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            if (gm && a.rmsnorm) {
                ld16(gm + (c * 32 + lane) * 8, gam[c]);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) gam[c][i] = 1.f;
            }
        }
        constexpr int HPW = NH / (kThreads / 32);  // heads per warp
        uint4 raw[HPW][CPL];
#pragma unroll
        for (int hi = 0; hi < HPW; ++hi)
#pragma unroll
            for (int c = 0; c < CPL; ++c)
                raw[hi][c] = __ldg(reinterpret_cast<const uint4*>(qg + (size_t)(warp * HPW + hi) * D) + c * 32 + lane);
        const int rope0 = D - a.rho;
#pragma unroll
        for (int hi = 0; hi < HPW; ++hi) {
            const int h = warp * HPW + hi;
            float x[CPL][8];
            float ss = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const uint32_t wv[4] = {raw[hi][c].x, raw[hi][c].y, raw[hi][c].z, raw[hi][c].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[c][2 * e] = __uint_as_float(wv[e] << 16);
                    x[c][2 * e + 1] = __uint_as_float(wv[e] & 0xffff0000u);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) ss = fmaf(x[c][i], x[c][i], ss);
            }
            if (a.rmsnorm) {
#pragma unroll
                for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
#pragma unroll
                for (int c = 0; c < CPL; ++c)
#pragma unroll
                    for (int i = 0; i < 8; ++i) x[c][i] *= inv * gam[c][i];
            }
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const int d0 = (c * 32 + lane) * 8;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (a.rho > 0 && d0 + 2 * e >= rope0)
                        rotate_pair(x[c][2 * e], x[c][2 * e + 1], cs[(d0 + 2 * e - rope0) >> 1]);
#pragma unroll
                for (int i = 0; i < 8; ++i) ovf |= fabsf(x[c][i]) > kF16Max;
                uint4 o;
                o.x = pack_f16x2(x[c][0], x[c][1]);
                o.y = pack_f16x2(x[c][2], x[c][3]);
                o.z = pack_f16x2(x[c][4], x[c][5]);
                o.w = pack_f16x2(x[c][6], x[c][7]);
                *reinterpret_cast<uint4*>(smem + Lay::OFF_Q + sw128_off(h, d0, Lay::QREG)) = o;
            }
        }
    }
    // this thread's own copies have landed: widen them to fp16 in place
    cp_async_wait_all();
    {
        constexpr int CPR = D / 8;
        for (int c = tid; c < n16 * CPR; c += kThreads) {
            const int row = c / CPR, ch = c % CPR;
            uint4* p = reinterpret_cast<uint4*>(smem + Lay::OFF_E + (uint32_t)(ch >> 3) * Lay::EREG +
                                                (uint32_t)(row >> 3) * 1024u + (uint32_t)(row & 7) * 128u +
                                                ((uint32_t)((ch & 7) ^ (row & 7)) << 4));
            uint4 u = *p;
            u.x = bf16x2_to_f16x2(u.x, ovf);
            u.y = bf16x2_to_f16x2(u.y, ovf);
            u.z = bf16x2_to_f16x2(u.z, ovf);
            u.w = bf16x2_to_f16x2(u.w, ovf);
            *p = u;
        }
    }
    fence_async_smem();
    if (__syncthreads_or(ovf) && tid == 0) set_status(a.status, LBCA_ERR_UNSUPPORTED);

    // ---- S^T = E . Q^T  (TMEM columns [0, NH), lane = entry row) ----
    const uint32_t sQ = smem_addr(smem + Lay::OFF_Q);
    const uint32_t sP = smem_addr(smem + Lay::OFF_P);
    if (tid == 0 && n > 0) {
        tc_fence_after();
        constexpr uint32_t idS = idesc_f16_f32(TE, NH, false);
#pragma unroll 4
        for (int kk = 0; kk < D / 16; ++kk)
            tc_mma_bf16(tbase, smem_desc_sw128(sE + (kk >> 2) * Lay::EREG + (kk & 3) * 32, 16, 1024),
                        smem_desc_sw128(sQ + (kk >> 2) * Lay::QREG + (kk & 3) * 32, 16, 1024), idS, kk > 0);
        tc_commit(&bars[0]);
    }

    // ---- per-head max and sum over this chunk; P^T (fp16) into shared memory ----
    // warp w reads TMEM lanes 32 (w & 3).. (entry rows) and heads 32 (w >> 2)..
    const int quad = warp & 3, hh = warp >> 2;
    const uint32_t lane_f = (uint32_t)(32 * quad) << 16;
    const int e = 32 * quad + lane;
    const bool valid = e < n;
    bool ok = true;
    if (n > 0) ok = mbar_wait(&bars[0], 0, kWaitNs);
    ok = __syncthreads_and(ok);
    if (!ok && tid == 0) set_status(a.status, LBCA_ERR_TIMEOUT);
    const bool live = ok && n > 0;
    const float sc = a.scale * kLog2e;
    float v[32];
    if (live) {
        tc_fence_after();
        tmem_ld32(tbase + lane_f + 32 * hh, v);
        tmem_wait_ld();
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = (live && valid) ? v[i] * sc : kNegInf;
    float s[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) s[i] = v[i];
    red[quad * NH + 32 * hh + lane] = warp_transpose_reduce<true>(v, lane);
    __syncthreads();
    if (tid < NH) {
        float M = red[tid];
#pragma unroll
        for (int q = 1; q < 4; ++q) M = fmaxf(M, red[q * NH + tid]);
        mh[tid] = M;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float M = mh[32 * hh + i];
        s[i] = (s[i] == kNegInf) ? 0.f : ex2(s[i] - M);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 o;
        o.x = pack_f16x2(s[8 * c + 0], s[8 * c + 1]);
        o.y = pack_f16x2(s[8 * c + 2], s[8 * c + 3]);
        o.z = pack_f16x2(s[8 * c + 4], s[8 * c + 5]);
        o.w = pack_f16x2(s[8 * c + 6], s[8 * c + 7]);
        *reinterpret_cast<uint4*>(smem + Lay::OFF_P + sw128_off(e, 32 * hh + 8 * c, 0)) = o;
    }
    fence_async_smem();
    red[4 * NH + quad * NH + 32 * hh + lane] = warp_transpose_reduce<false>(s, lane);
    __syncthreads();
    if (tid < NH) {
        float l = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) l += red[4 * NH + q * NH + tid];
        ml[tid] = mh[tid];
        ml[NH + tid] = l;
    }

    // ---- O^T = E^T . P^T  (TMEM columns [NH + NH mt, ...), lane = dim within tile mt) ----
    if (tid == 0 && live) {
        tc_fence_after();
        constexpr uint32_t idO = idesc_f16_f32_mn_mn(128, NH);
        for (int mt = 0; mt < D / 128; ++mt)
            for (int kk = 0; kk < n16 / 16; ++kk)
                tc_mma_bf16(tbase + NH + NH * mt, smem_desc_sw128(sE + 2 * mt * Lay::EREG + kk * 2048, Lay::EREG, 1024),
                            smem_desc_sw128(sP + kk * 2048, Lay::EREG, 1024), idO, kk > 0);
        tc_commit(&bars[1]);
    }
    bool ok2 = true;
    if (live) ok2 = mbar_wait(&bars[1], 0, kWaitNs);
    ok2 = __syncthreads_and(ok2);
    if (!ok2 && tid == 0) set_status(a.status, LBCA_ERR_TIMEOUT);
    const bool have_o = live && ok2;
    tc_fence_after();
    fence_async_smem();  // E and Q are rewritten by the generic-proxy merge below

    // ---- merge across the cluster ----
    cluster.sync();  // every CTA's (max, sum) published; every CTA's MMAs have read E
    if (tid < NH) {
        const int hg = g * NH + tid;
        float Ms[16], Ls[16];
        float M = kNegInf;
        for (int r = 0; r < CS; ++r) {
            const float* rm = cluster.map_shared_rank(ml, r);
            Ms[r] = rm[tid];
            Ls[r] = rm[NH + tid];
            M = fmaxf(M, Ms[r]);
        }
        const float sk = a.sink ? a.sink[hg] * kLog2e : kNegInf;
        M = fmaxf(M, sk);
        float den = 0.f;
        if (M != kNegInf) {
            for (int r = 0; r < CS; ++r) den = fmaf(Ls[r], Ms[r] == kNegInf ? 0.f : ex2(Ms[r] - M), den);
            if (a.sink) den += ex2(sk - M);
        }
        const float mine = ml[tid];
        fh[tid] = (den > 0.f && mine != kNegInf) ? ex2(mine - M) / den : 0.f;
    }
    __syncthreads();
    // push this CTA's scaled O^T slices: dim d goes to rank d / SW
#pragma unroll 1
    for (int mt = 0; mt < D / 128; ++mt) {
        if (have_o) {
            tmem_ld32(tbase + lane_f + NH + NH * mt + 32 * hh, v);
            tmem_wait_ld();
        }
        const int d = 128 * mt + 32 * quad + lane;
        const int owner = d / SW, dd = d % SW;
        float* dst = cluster.map_shared_rank(recv, owner);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int h4 = 8 * hh + j;  // heads 4 h4 .. 4 h4 + 3
            float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
            if (have_o) {
                o.x = v[4 * j + 0] * fh[4 * h4 + 0];
                o.y = v[4 * j + 1] * fh[4 * h4 + 1];
                o.z = v[4 * j + 2] * fh[4 * h4 + 2];
                o.w = v[4 * j + 3] * fh[4 * h4 + 3];
            }
            *reinterpret_cast<float4*>(dst + (((size_t)rank * (NH / 4) + h4) * SW + dd) * 4) = o;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, Lay::TMEM_COLS);
    cluster.sync();  // every slice has landed; nothing remote is touched after this

    // ---- sum the slices, turn the rotated dims back by -t, write bf16 ----
    const int rope0 = D - a.rho;
    __nv_bfloat16* outp = static_cast<__nv_bfloat16*>(a.out) + ((size_t)b * a.Hq + (size_t)g * NH) * D;
    for (int u = tid; u < SW * (NH / 4); u += kThreads) {  // SW * 16 is a multiple of 256: no divergence
        const int dd = u % SW, h4 = u / SW;
        const int d = rank * SW + dd;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < CS; ++r) {
            const float4 x = *reinterpret_cast<const float4*>(recv + (((size_t)r * (NH / 4) + h4) * SW + dd) * 4);
            acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
        }
        float4 p;  // the pair partner: pairs (d, d + 1) sit in lanes (2i, 2i + 1)
        p.x = __shfl_xor_sync(0xffffffffu, acc.x, 1);
        p.y = __shfl_xor_sync(0xffffffffu, acc.y, 1);
        p.z = __shfl_xor_sync(0xffffffffu, acc.z, 1);
        p.w = __shfl_xor_sync(0xffffffffu, acc.w, 1);
        if (a.shared && a.rho > 0 && d >= rope0) {
            const float2 c = cs[(d - rope0) >> 1];
            if ((d & 1) == 0) {  // x' = x c + y s
                acc.x = acc.x * c.x + p.x * c.y; acc.y = acc.y * c.x + p.y * c.y;
                acc.z = acc.z * c.x + p.z * c.y; acc.w = acc.w * c.x + p.w * c.y;
            } else {             // y' = y c - x s
                acc.x = acc.x * c.x - p.x * c.y; acc.y = acc.y * c.x - p.y * c.y;
                acc.z = acc.z * c.x - p.z * c.y; acc.w = acc.w * c.x - p.w * c.y;
            }
        }
        outp[(size_t)(4 * h4 + 0) * D + d] = __float2bfloat16_rn(acc.x);
        outp[(size_t)(4 * h4 + 1) * D + d] = __float2bfloat16_rn(acc.y);
        outp[(size_t)(4 * h4 + 2) * D + d] = __float2bfloat16_rn(acc.z);
        outp[(size_t)(4 * h4 + 3) * D + d] = __float2bfloat16_rn(acc.w);
    }
}

// Largest cluster size (16, else 8) this kernel can be scheduled with, cached.
template <int D>
int max_cluster() {
    static int best = -1;
    if (best >= 0) return best;
    auto fn = decode_mqa_tc_kernel<D>;
    best = 0;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, MqaLayout<D>::SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        return best;
    }
    for (int cs : {16, 8, 4, 2, 1}) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(cs, 1, 1);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = MqaLayout<D>::SMEM;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclu = 0;
        if (cudaOccupancyMaxActiveClusters(&nclu, fn, &cfg) == cudaSuccess && nclu > 0) {
            best = cs;
            break;
        }
        cudaGetLastError();
    }
    return best;
}

template <int D>
cudaError_t launch_d(const DecodeArgs& a, cudaStream_t s) {
    auto fn = decode_mqa_tc_kernel<D>;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.tc_cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(a.tc_cs, a.G, a.B);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = MqaLayout<D>::SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fn, a);
}

}  // namespace

int plan_decode_mqa_tc(int dtype, int B, int Hq, int G, int D, int m, int w, int shared, int max_ctx) {
    if (dtype != LBCA_BF16 || !shared || G < 1 || Hq != NH * G || (D != 256 && D != 512)) return 0;
    if (B < 1 || max_ctx < 1) return 0;
    const long long P = max_ctx - w > 0 ? (long long)(max_ctx - w) / m : 0;
    const long long max_vis = std::min<long long>(max_ctx, P + w + m - 1);
    const int cap = D == 512 ? max_cluster<512>() : max_cluster<256>();
    int cs = 1;
    while ((long long)cs * TE < max_vis) cs *= 2;
    if (cs > cap) return 0;
    while (cs < cap && (long long)B * G * cs < 148) cs *= 2;  // spread short batches over the SMs
    return cs;
}

cudaError_t launch_decode_mqa_tc(const DecodeArgs& a, cudaStream_t s) {
    if (a.B == 0) return cudaSuccess;
    if (a.D == 512) return launch_d<512>(a, s);
    if (a.D == 256) return launch_d<256>(a, s);
    return cudaErrorInvalidValue;
}

}  // namespace lbca
