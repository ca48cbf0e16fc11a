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
// B200 mapping: grid (CS, G, B), cluster (CS, 1, 1), 16 warps per CTA.  The CS
// CTAs of a cluster share one (sequence, kv head):
//   1. Each CTA copies its chunk of the visible list (<= C rows: pooled rows,
//      then ring rows) into 128-byte-swizzled shared memory with 16-byte
//      cp.async and widens it to fp16 in place.  The ring holds the raw
//      entries as appended; a warp finalises each of them (RMSNorm, RoPE at
//      the token's position) in f32 before its one fp16 rounding, so a window
//      row that is also the value carries no bf16 rounding of its own.  Meanwhile up to 8 CTAs each
//      prepare a share of the queries (RMSNorm, RoPE at t, fp16) and
//      bulk-copy it into every other CTA's query tile (shared memory to
//      shared memory across the cluster, one destination per copy).
//   2. One thread issues S^T; warps take each head's max over the chunk with
//      a transposing butterfly, and every CTA pushes its maxima to all CTAs.
//      After one cluster barrier every CTA holds the same per-head reference
//      max M (the sink included), so the CTAs' partial outputs share one
//      scale and simply add.
//   3. P = 2^(s - M) (fp16) -> P^T tile; per-head sums; O^T on tcgen05.
//   4. Each CTA rounds its O^T to fp16, lays it out by owner (dims
//      [r SW, (r+1) SW) belong to CTA r) and bulk-copies one slice, plus its
//      sums, to each owner.  An owner waits for its CS slices on an mbarrier,
//      adds them, divides by the summed sums plus the sink term, turns the
//      rotated dims back by -t and writes bf16.
// A sequence whose whole visible list fits one chunk skips the exchange: its
// first CTA takes every entry and writes the output straight from TMEM.
//
// Serving step (append fused, one kv head): the new token is cached first and
// the query attends at the new length L = cached + 1 (mSeek README, "How LBCA
// works", steps 2-4).  Its raw entry is the last visible row, so the CTA
// whose chunk ends the list appends it with one warp while the other rows'
// copies are in flight: running per-channel softmax of the open block (and the
// finished pooled entry when the token closes a block), the raw row to the
// ring and straight into its own staged tile, where it is finalised with the
// other window rows.  With a window (n_win > 0) a block closed at this step is
// not yet visible, so no other CTA needs what the append writes.  The arithmetic and its order are
// those of the stand-alone append kernel, so the cache and the output are
// bit-identical to append followed by decode.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace lbca {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int NH = 64;          // query heads per kv head (N of both MMAs)
constexpr int NGRP = NH / 8;    // 8-head groups of the query tile
constexpr int kMaxCS = 16;
constexpr uint64_t kWaitNs = 200ull * 1000 * 1000;

// Output dims owned by each CTA of a CS-CTA cluster (even, so RoPE pairs never split).
__host__ __device__ inline int owned_dims(int D, int CS) { return ((D + CS - 1) / CS + 1) & ~1; }

// Shared-memory plan for head dim D, C entry rows per CTA (a multiple of 16, <= 128)
// and CS CTAs per cluster.
struct MqaLayout {
    uint32_t EREG, GS, SLICE;
    uint32_t OFF_E, OFF_Q, OFF_P, OFF_MALL, OFF_LRECV, OFF_CS, OFF_TURN, OFF_RED, OFF_MH, OFF_LLOC, OFF_DEN, OFF_BAR;
    uint32_t TOTAL, SMEM;
    __host__ __device__ MqaLayout(int D, int C, int CS) {
        EREG = (uint32_t)C * 128u;                          // one 64-dim column region of E
        GS = (uint32_t)(D / 64) * 1024u;                    // one 8-head group of Q (all regions)
        SLICE = (uint32_t)(NH / 4) * owned_dims(D, CS) * 8u;  // fp16 [NH/4][SW][4] per owner
        const uint32_t e_bytes = (uint32_t)(D / 64) * EREG;
        const uint32_t xfer = (uint32_t)CS * SLICE;          // O^T staging (aliases E) / receive (aliases Q)
        const uint32_t q_bytes = (uint32_t)NH * D * 2u;
        OFF_E = 0;
        OFF_Q = ((e_bytes > xfer ? e_bytes : xfer) + 1023u) & ~1023u;
        OFF_P = (OFF_Q + (q_bytes > xfer ? q_bytes : xfer) + 1023u) & ~1023u;
        OFF_MALL = OFF_P + (uint32_t)C * 128u;              // [kMaxCS][NH] f32 pushed maxima
        OFF_LRECV = OFF_MALL + kMaxCS * NH * 4u;            // [kMaxCS][NH] f32 pushed sums
        OFF_CS = OFF_LRECV + kMaxCS * NH * 4u;              // [D/2] float2 cos/sin at t
        OFF_TURN = OFF_CS + (uint32_t)(D / 2) * 8u;         // [D/2] u64 fixed-point turns per position
        OFF_RED = OFF_TURN + (uint32_t)(D / 2) * 8u;        // [4][NH] warp partials
        OFF_MH = OFF_RED + 4u * NH * 4u;                    // [NH] reference max
        OFF_LLOC = OFF_MH + NH * 4u;                        // [NH] this CTA's sums
        OFF_DEN = OFF_LLOC + NH * 4u;                       // [NH] denominators
        OFF_BAR = OFF_DEN + NH * 4u;                        // 4 mbarriers + TMEM base
        TOTAL = OFF_BAR + 64u;
        SMEM = TOTAL + 1024u;                               // slack for 1024-byte alignment
    }
};


// Butterfly over the 32 lanes of a warp for 16 values per lane: lane l ends up
// holding the reduction over all 32 lanes of v[l % 16] (16 shuffles).
template <bool kMax>
__device__ __forceinline__ float warp_transpose_reduce16(float (&v)[16], int lane) {
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float send = up ? v[i] : v[i + o];
            const float keep = up ? v[i + o] : v[i];
            const float got = __shfl_xor_sync(0xffffffffu, send, o);
            v[i] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
    const float got = __shfl_xor_sync(0xffffffffu, v[0], 16);
    return kMax ? fmaxf(v[0], got) : v[0] + got;
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

__device__ __forceinline__ float2 unpack_f16x2(uint32_t w) {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    return __half22float2(h);
}

// Sequential sum over the warp of each lane's CPL values, in chunk order
// (chunk c * 32 + lane holds v[c]): the order of the stand-alone append's
// per-head sum, so both give the same bits.
template <int CPL>
__device__ __forceinline__ float chunk_order_sum(const float (&v)[CPL]) {
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c)
#pragma unroll
        for (int src = 0; src < 32; ++src) s += __shfl_sync(0xffffffffu, v[c], src);
    return s;
}

// RMSNorm (when on) and RoPE of one lane's chunks of a finished entry; cos/sin
// from `cs` (pairs from dim D - rho on) or, when it is null, at position `rpos`.
template <int D, int CPL>
__device__ __forceinline__ void finalise_row(const DecodeArgs& a, float (&e)[CPL][8], int lane, const float2* cs,
                                             int64_t rpos) {
    if (a.rmsnorm) {
        float v[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            v[c] = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) v[c] += e[c][k] * e[c][k];
        }
        const float ss = chunk_order_sum<CPL>(v);
        const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
        const __nv_bfloat16* gm = static_cast<const __nv_bfloat16*>(a.gamma_kv);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            float gam[8];
            if (gm) {
                ld16(gm + (c * 32 + lane) * 8, gam);
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) gam[k] = 1.0f;
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) e[c][k] *= inv * gam[k];
        }
    }
    if (a.rho) {
        const int base = D - a.rho;
#pragma unroll
        for (int c = 0; c < CPL; ++c)
#pragma unroll
            for (int k = 0; k < 8; k += 2) {
                const int d = (c * 32 + lane) * 8 + k;
                if (d >= base) {
                    const int kk = (d - base) >> 1;
                    rotate_pair(e[c][k], e[c][k + 1], cs ? cs[kk] : rope_cs(rpos, kk, a.rope_step));
                }
            }
    }
}

// The fused append of the new token at `pos` for (sequence b, kv head g), by
// one warp: lane l owns the 16-byte chunks l, l + 32, ... of the D-dim row.
// The running per-channel softmax of the open block (max, sum and weighted
// sum in the log2 domain, the B_pos row of the token's offset) is advanced;
// a token that closes block j finishes entry j (weighted sum / sum, RMSNorm,
// RoPE at the block start j m) into pooled_k, otherwise the state is stored
// back; the raw token (RMSNorm, RoPE at pos, from `cs_t`) goes to its ring
// slot and, when `row` >= 0, to that row of the staged bf16 entry tile, as
// given: window rows are finalised when the tile is widened.
template <int D>
__device__ __forceinline__ void append_token(const DecodeArgs& a, int b, int g, int pos, uint8_t* sE, uint32_t ereg,
                                             int row, int lane) {
    constexpr int CPL = D / 256;
    const int GD = a.G * D;
    const int i = pos % a.m, jb = pos / a.m;
    const size_t tok = ((size_t)b * a.G + g) * D;
    const __nv_bfloat16* xk = static_cast<const __nv_bfloat16*>(a.app_k) + tok;
    const __nv_bfloat16* zk = static_cast<const __nv_bfloat16*>(a.app_z) + tok;
    const __nv_bfloat16* bp = static_cast<const __nv_bfloat16*>(a.app_bp) + (size_t)i * GD + (size_t)g * D;
    float* st = a.state + (size_t)b * 3 * GD + (size_t)g * D;
    float x[CPL][8], mx[CPL][8], l[CPL][8], acc[CPL][8];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int d0 = (c * 32 + lane) * 8;
        float z[8], bpv[8];
        ld16(xk + d0, x[c]);
        ld16(zk + d0, z);
        ld16(bp + d0, bpv);
        float m0[8], l0[8], a0[8];
        if (i > 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float4 u = *reinterpret_cast<const float4*>(st + d0 + 4 * h);
                const float4 w = *reinterpret_cast<const float4*>(st + GD + d0 + 4 * h);
                const float4 y = *reinterpret_cast<const float4*>(st + 2 * GD + d0 + 4 * h);
                m0[4 * h] = u.x; m0[4 * h + 1] = u.y; m0[4 * h + 2] = u.z; m0[4 * h + 3] = u.w;
                l0[4 * h] = w.x; l0[4 * h + 1] = w.y; l0[4 * h + 2] = w.z; l0[4 * h + 3] = w.w;
                a0[4 * h] = y.x; a0[4 * h + 1] = y.y; a0[4 * h + 2] = y.z; a0[4 * h + 3] = y.w;
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float av = (z[e] + bpv[e]) * kLog2e;
            if (i == 0) {
                mx[c][e] = av; l[c][e] = 1.f; acc[c][e] = x[c][e];
            } else {
                const float mn = fmaxf(m0[e], av);
                const float r = ex2(m0[e] - mn), p = ex2(av - mn);
                mx[c][e] = mn;
                l[c][e] = l0[e] * r + p;
                acc[c][e] = fmaf(p, x[c][e], a0[e] * r);
            }
        }
    }
    if (i == a.m - 1) {  // the token closes block jb
        float e[CPL][8];
#pragma unroll
        for (int c = 0; c < CPL; ++c)
#pragma unroll
            for (int k = 0; k < 8; ++k) e[c][k] = acc[c][k] / l[c][k];
        finalise_row<D, CPL>(a, e, lane, nullptr, (int64_t)jb * a.m);
        if (jb < a.max_blocks) {
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.pooled_w) + (((size_t)b * a.G + g) * a.max_blocks + jb) * D;
#pragma unroll
            for (int c = 0; c < CPL; ++c) st16(o + (c * 32 + lane) * 8, e[c]);
        } else if (lane == 0) {
            set_status(a.status, LBCA_ERR_CAPACITY);
        }
    } else {
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int d0 = (c * 32 + lane) * 8;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                *reinterpret_cast<float4*>(st + d0 + 4 * h) =
                    make_float4(mx[c][4 * h], mx[c][4 * h + 1], mx[c][4 * h + 2], mx[c][4 * h + 3]);
                *reinterpret_cast<float4*>(st + GD + d0 + 4 * h) =
                    make_float4(l[c][4 * h], l[c][4 * h + 1], l[c][4 * h + 2], l[c][4 * h + 3]);
                *reinterpret_cast<float4*>(st + 2 * GD + d0 + 4 * h) =
                    make_float4(acc[c][4 * h], acc[c][4 * h + 1], acc[c][4 * h + 2], acc[c][4 * h + 3]);
            }
        }
    }
    // the raw entry as given joins the window (ring slot and staged tile row);
    // like every window row it is finalised when the tile is widened
    __nv_bfloat16* ring = static_cast<__nv_bfloat16*>(a.ring_w) + (((size_t)b * a.G + g) * a.R + pos % a.R) * D;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int ch = c * 32 + lane;
        uint4 u;
        u.x = pack_bf16x2(x[c][0], x[c][1]);
        u.y = pack_bf16x2(x[c][2], x[c][3]);
        u.z = pack_bf16x2(x[c][4], x[c][5]);
        u.w = pack_bf16x2(x[c][6], x[c][7]);
        *reinterpret_cast<uint4*>(ring + ch * 8) = u;
        if (row >= 0)
            *reinterpret_cast<uint4*>(sE + (uint32_t)(row >> 3) * 1024u + (uint32_t)(row & 7) * 128u +
                                      (uint32_t)(ch >> 3) * ereg + ((uint32_t)((ch & 7) ^ (row & 7)) << 4)) = u;
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) decode_mqa_tc_kernel(const DecodeArgs a) {
    constexpr int CPR = D / 8;    // 16-byte chunks per entry row
    constexpr int CPL = D / 256;  // 16-byte query chunks per lane per head
    static_assert(D % 256 == 0 && D <= 512, "D must be 256 or 512");
    const int C = a.chunk;        // entry rows per CTA (multiple of 16, <= 128)
    const int CS = a.tc_cs;
    const MqaLayout lay(D, C, CS);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + lay.OFF_BAR);  // S done, O done, Q in, slices in
    uint32_t* tmem_sh = reinterpret_cast<uint32_t*>(smem + lay.OFF_BAR + 32);
    float2* cs = reinterpret_cast<float2*>(smem + lay.OFF_CS);
    uint64_t* turns = reinterpret_cast<uint64_t*>(smem + lay.OFF_TURN);
    float* red = reinterpret_cast<float*>(smem + lay.OFF_RED);
    float* mh = reinterpret_cast<float*>(smem + lay.OFF_MH);
    float* lloc = reinterpret_cast<float*>(smem + lay.OFF_LLOC);
    float* den = reinterpret_cast<float*>(smem + lay.OFF_DEN);
    const float* mall = reinterpret_cast<const float*>(smem + lay.OFF_MALL);
    const float* lrecv = reinterpret_cast<const float*>(smem + lay.OFF_LRECV);

    const int rank = (int)blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, hq = warp >> 2;  // TMEM lane quarter, head group of 16
    const int SW = owned_dims(D, CS);

    // ---- visible set of this sequence (block-aligned partition) and this CTA's chunk ----
    const bool fuse = a.app_k != nullptr;
    const int pos = a.seq_lens[b];  // cached tokens (fused: the new token's position)
    const int L = fuse ? pos + 1 : pos;
    const int t = L - 1;
    // the visible list: P pooled entries, then the raw window tokens [s0, t]
    // (block-aligned partition); with a selection (CSA form) the selected
    // entries, then the window of the last n_win tokens, which may cover
    // tokens a selected entry also summarises
    int P, s0, n_vis;
    if (a.sel) {
        P = L > 0 ? min(a.sel_k, min(L / a.m, a.max_blocks)) : 0;
        const int nw = min(L, a.w);
        s0 = L - nw;
        n_vis = L > 0 ? P + nw : 0;
        if (nw > a.R || n_vis > C * CS) {
            if (rank == 0 && g == 0 && tid == 0) set_status(a.status, LBCA_ERR_CAPACITY);
            n_vis = 0;
        }
    } else {
        P = visible_blocks(L, a.m, a.w);
        s0 = P * a.m;
        n_vis = L > 0 ? P + (L - s0) : 0;
        if (P > a.max_blocks || L - s0 > a.R || n_vis > C * CS) {  // cache or split grid cannot hold it
            if (rank == 0 && g == 0 && tid == 0) set_status(a.status, LBCA_ERR_CAPACITY);
            n_vis = 0;
        }
    }
    const bool single = n_vis <= C;  // one CTA takes the whole list: no exchange (uniform per cluster)
    const int chunk = single ? n_vis : (n_vis + CS - 1) / CS;
    const int e0 = single ? 0 : rank * chunk;
    const int n = single ? (rank == 0 ? n_vis : 0) : max(0, min(n_vis, e0 + chunk) - e0);
    const int n16 = (n + 15) & ~15;
    // fused append: the CTA holding the last visible row (the new token), the
    // warp that would have copied that row; row -1 when nothing is visible
    const int app_rank = (n_vis == 0 || single) ? 0 : (n_vis - 1) / chunk;
    const bool appender = fuse && rank == app_rank;
    const int app_row = (appender && n_vis > 0) ? n_vis - 1 - e0 : -1;
    const int app_warp = app_row >= 0 ? app_row % kWarps : 0;

    // query groups this CTA prepares for the whole cluster
    const int preppers = CS >= 8 ? 8 : (CS >= 4 ? 4 : (CS >= 2 ? 2 : 1));
    const int gpc = NGRP / preppers;
    const bool prepper = rank < preppers;
    const uint32_t my_q_bytes = prepper ? (uint32_t)gpc * lay.GS : 0u;

    const uint32_t sE = smem_addr(smem + lay.OFF_E), sQ = smem_addr(smem + lay.OFF_Q);
    const uint32_t sP = smem_addr(smem + lay.OFF_P);
    const uint32_t bar_q = smem_addr(&bars[2]), bar_r = smem_addr(&bars[3]);

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        fence_barrier_init();
        mbar_arrive_expect_tx(&bars[2], (uint32_t)NH * D * 2u - my_q_bytes);
        mbar_arrive_expect_tx(&bars[3], single ? 0u : (uint32_t)CS * (lay.SLICE + NH * 4u));
    }
    __syncwarp();
    if (warp == 0) tmem_alloc(tmem_sh, 512);
    cluster_arrive_relaxed();  // this CTA's barriers exist (waited for before the first push)

    // ---- stage the chunk's entry rows (bf16), 128-byte swizzled; rows [n, n16) zero ----
    const size_t pool_head = ((size_t)b * a.G + g) * a.max_blocks;
    const size_t ring_head = ((size_t)b * a.G + g) * a.R;
    const __nv_bfloat16* pk = static_cast<const __nv_bfloat16*>(a.pooled_k);
    const __nv_bfloat16* rk = static_cast<const __nv_bfloat16*>(a.ring_k);
    for (int row = warp; row < n16; row += kWarps) {
        if (row == app_row) continue;  // the new token: written below by this warp
        const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(a.q);  // any valid address (zero fill)
        uint32_t bytes = 0;
        if (row < n) {
            const int idx = e0 + row;
            bytes = 16;
            if (idx < P) {
                int j = idx;
                if (a.sel) {  // a selected entry: its index must name a stored block
                    j = a.sel[(size_t)b * a.sel_k + idx];
                    if (j < 0 || j >= a.max_blocks) {
                        if (lane == 0) set_status(a.status, LBCA_ERR_ARG);
                        j = 0;
                        bytes = 0;  // zero row
                    }
                }
                src = pk + (pool_head + checked_rows(j, 1, a.max_blocks, a.status)) * D;
            } else {
                src = rk + (ring_head + checked_rows((s0 + (idx - P)) % a.R, 1, a.R, a.status)) * D;
            }
        }
        const uint32_t rbase = sE + (uint32_t)(row >> 3) * 1024u + (uint32_t)(row & 7) * 128u;
#pragma unroll
        for (int j = 0; j < CPR / 32; ++j) {
            const int ch = j * 32 + lane;
            cp_async16(rbase + (uint32_t)(ch >> 3) * lay.EREG + ((uint32_t)((ch & 7) ^ (row & 7)) << 4),
                       bytes ? src + ch * 8 : src, bytes);
        }
    }

    // ---- cos/sin at t; this CTA's query groups: RMSNorm, RoPE, fp16, group-major swizzled ----
    for (int k = tid; k < a.rho / 2; k += kThreads) {
        const uint64_t F = rope_turns(k, a.rope_step);
        turns[k] = F;
        cs[k] = rope_cs_turns((int64_t)t, F);
    }
    // the query and the new token may come from the preceding kernel (programmatic
    // dependent launch): everything above reads only this cache
    griddep_wait();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_sh;
    bool ovf = false;
    if (prepper) {
        const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q) + ((size_t)b * a.Hq + (size_t)g * NH) * D;
        const __nv_bfloat16* gm = static_cast<const __nv_bfloat16*>(a.gamma_q);
        const int rope0 = D - a.rho;
        for (int hi = warp; hi < gpc * 8; hi += kWarps) {
            const int h = rank * gpc * 8 + hi;
            float x[CPL][8];
            float ss = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                ld16(qg + (size_t)h * D + (c * 32 + lane) * 8, x[c]);
#pragma unroll
                for (int i = 0; i < 8; ++i) ss = fmaf(x[c][i], x[c][i], ss);
            }
            if (a.rmsnorm) {
#pragma unroll
                for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    float gam[8];
                    if (gm) {
                        ld16(gm + (c * 32 + lane) * 8, gam);
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i) gam[i] = 1.f;
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) x[c][i] *= inv * gam[i];
                }
            }
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const int ch = c * 32 + lane, d0 = ch * 8;
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
                const int hr = h & 7;
                *reinterpret_cast<uint4*>(smem + lay.OFF_Q + (uint32_t)(h >> 3) * lay.GS + (uint32_t)(ch >> 3) * 1024u +
                                          (uint32_t)hr * 128u + ((uint32_t)((ch & 7) ^ hr) << 4)) = o;
            }
        }
        fence_async_smem();
    }
    if (appender && warp == app_warp) append_token<D>(a, b, g, pos, smem + lay.OFF_E, lay.EREG, app_row, lane);
    __syncthreads();
    cluster_wait_acquire();  // every CTA's barriers exist; every CTA has read seq_lens[b]
    if (appender && tid == 0) a.lens_w[b] = pos + 1;
    const bool q_sender = prepper && tid < CS && tid != rank;
    if (q_sender) {  // this CTA's query groups to CTA `tid`
        for (int G = rank * gpc; G < rank * gpc + gpc; ++G) {
            const uint32_t off = sQ + (uint32_t)G * lay.GS;
            bulk_to_peer(peer_addr(off, tid), off, lay.GS, peer_addr(bar_q, tid));
        }
        bulk_commit();
    }

    // ---- this thread's entry copies have landed: widen them to fp16 in place.
    // Pooled rows are finalised entries; window rows are the raw entries as
    // appended and are finalised here, in f32 (RMSNorm over the row held by
    // this warp, RoPE at the token's position), before their one fp16 rounding.
    cp_async_wait_all();
    for (int row = warp; row < n16; row += kWarps) {
        uint8_t* rbase = smem + lay.OFF_E + (uint32_t)(row >> 3) * 1024u + (uint32_t)(row & 7) * 128u;
        const int idx = e0 + row;
        if (row < n && idx >= P) {  // uniform per warp: a window row
            float x[CPR / 32][8];
            float ss = 0.f;
#pragma unroll
            for (int j = 0; j < CPR / 32; ++j) {
                const int ch = j * 32 + lane;
                const uint4 u = *reinterpret_cast<const uint4*>(rbase + (uint32_t)(ch >> 3) * lay.EREG +
                                                                ((uint32_t)((ch & 7) ^ (row & 7)) << 4));
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    x[j][2 * i] = __uint_as_float(w[i] << 16);
                    x[j][2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) ss = fmaf(x[j][i], x[j][i], ss);
            }
            if (a.rmsnorm) {
#pragma unroll
                for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
                const __nv_bfloat16* gm = static_cast<const __nv_bfloat16*>(a.gamma_kv);
#pragma unroll
                for (int j = 0; j < CPR / 32; ++j) {
                    float gam[8];
                    if (gm) {
                        ld16(gm + (j * 32 + lane) * 8, gam);
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i) gam[i] = 1.f;
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) x[j][i] *= inv * gam[i];
                }
            }
            // RoPE at the token's position: lane l forms cos/sin of pair kb + l
            // (one sincos per lane for 32 pairs), the lanes holding a pair's
            // dims take it by shuffle
            const int64_t spos = (int64_t)s0 + (idx - P);
            const int rope0 = D - a.rho;
            for (int kb = 0; kb < a.rho / 2; kb += 32) {
                const int k = kb + lane;
                const float2 mine = k < a.rho / 2 ? rope_cs_turns(spos, turns[k]) : make_float2(1.f, 0.f);
#pragma unroll
                for (int j = 0; j < CPR / 32; ++j) {
                    const int ch = j * 32 + lane;
#pragma unroll
                    for (int i = 0; i < 8; i += 2) {
                        const int kk = (ch * 8 + i - rope0) >> 1;  // this lane's pair (negative: not rotated)
                        const bool here = ch * 8 + i >= rope0 && kk >= kb && kk < kb + 32;
                        const int src = here ? kk - kb : lane;
                        const float2 c = make_float2(__shfl_sync(0xffffffffu, mine.x, src),
                                                     __shfl_sync(0xffffffffu, mine.y, src));
                        if (here) rotate_pair(x[j][i], x[j][i + 1], c);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < CPR / 32; ++j) {
                const int ch = j * 32 + lane;
#pragma unroll
                for (int i = 0; i < 8; ++i) ovf |= fabsf(x[j][i]) > kF16Max;
                uint4 o;
                o.x = pack_f16x2(x[j][0], x[j][1]);
                o.y = pack_f16x2(x[j][2], x[j][3]);
                o.z = pack_f16x2(x[j][4], x[j][5]);
                o.w = pack_f16x2(x[j][6], x[j][7]);
                *reinterpret_cast<uint4*>(rbase + (uint32_t)(ch >> 3) * lay.EREG +
                                          ((uint32_t)((ch & 7) ^ (row & 7)) << 4)) = o;
            }
            continue;
        }
#pragma unroll
        for (int j = 0; j < CPR / 32; ++j) {
            const int ch = j * 32 + lane;
            uint4* p = reinterpret_cast<uint4*>(rbase + (uint32_t)(ch >> 3) * lay.EREG +
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

    // ---- the other CTAs' query groups, then S^T = E . Q^T (TMEM columns [0, NH)) ----
    bool ok = true;
    if (tid == 0) ok = mbar_wait(&bars[2], 0, kWaitNs);
    ok = __syncthreads_and(ok);
    if (tid == 0 && ok && n > 0) {
        tc_fence_after();
        constexpr uint32_t idS = idesc_f16_f32(128, NH, false);
#pragma unroll 4
        for (int kk = 0; kk < D / 16; ++kk)
            tc_mma_bf16(tbase, smem_desc_sw128(sE + (kk >> 2) * lay.EREG + (kk & 3) * 32, 16, 1024),
                        smem_desc_sw128(sQ + (kk >> 2) * 1024 + (kk & 3) * 32, 16, lay.GS), idS, kk > 0);
        tc_commit(&bars[0]);
    }
    if (ok && n > 0 && tid == 0) ok = mbar_wait(&bars[0], 0, kWaitNs);
    ok = __syncthreads_and(ok);
    if (!ok && tid == 0) set_status(a.status, LBCA_ERR_TIMEOUT);
    const bool live = ok && n > 0;

    // ---- per-head max over this chunk; warp (quad, hq) holds entry rows 32 quad.. x heads 16 hq.. ----
    const uint32_t lane_f = (uint32_t)(32 * quad) << 16;
    const int e = 32 * quad + lane;
    const bool valid = e < n;
    const float sc = a.scale * kLog2e;
    float s[16];
    if (live) {
        tc_fence_after();
        tmem_ld16(tbase + lane_f + 16 * hq, s);
        tmem_wait_ld();
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) s[i] = (live && valid) ? s[i] * sc : kNegInf;
    {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = s[i];
        const float r = warp_transpose_reduce16<true>(v, lane);
        if (lane < 16) red[quad * NH + 16 * hq + lane] = r;
    }
    __syncthreads();
    const float sink_l2 = (a.sink && tid < NH) ? a.sink[g * NH + tid] * kLog2e : kNegInf;
    if (tid < NH) {
        const float m = fmaxf(fmaxf(red[tid], red[NH + tid]), fmaxf(red[2 * NH + tid], red[3 * NH + tid]));
        if (single) {
            mh[tid] = fmaxf(m, sink_l2);
        } else {
            const uint32_t dst = smem_addr(smem + lay.OFF_MALL) + (uint32_t)(rank * NH + tid) * 4u;
            for (int r = 0; r < CS; ++r) st_peer_f32(peer_addr(dst, r), m);
        }
    }
    if (q_sender) bulk_wait_read_all();  // the query tile is overwritten by the slices below
    if (!single) {
        cluster_arrive_release();
        cluster_wait_acquire();  // every CTA's maxima have landed everywhere; every S^T is done
        if (tid < NH) {
            float m = sink_l2;
            for (int r = 0; r < CS; ++r) m = fmaxf(m, mall[r * NH + tid]);
            mh[tid] = m;
        }
    }
    __syncthreads();

    // ---- P = 2^(s - M) (fp16) into the P^T tile; per-head sums ----
#pragma unroll
    for (int i = 0; i < 16; ++i) s[i] = s[i] == kNegInf ? 0.f : ex2(s[i] - mh[16 * hq + i]);
    if (e < C) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint4 o;
            o.x = pack_f16x2(s[8 * c + 0], s[8 * c + 1]);
            o.y = pack_f16x2(s[8 * c + 2], s[8 * c + 3]);
            o.z = pack_f16x2(s[8 * c + 4], s[8 * c + 5]);
            o.w = pack_f16x2(s[8 * c + 6], s[8 * c + 7]);
            *reinterpret_cast<uint4*>(smem + lay.OFF_P + sw128_off(e, 16 * hq + 8 * c, 0)) = o;
        }
    }
    fence_async_smem();
    {
        const float r = warp_transpose_reduce16<false>(s, lane);
        if (lane < 16) red[quad * NH + 16 * hq + lane] = r;
    }
    __syncthreads();
    if (tid < NH) lloc[tid] = red[tid] + red[NH + tid] + red[2 * NH + tid] + red[3 * NH + tid];

    // ---- O^T = E^T . P^T (TMEM columns [NH + NH mt, ...), lane = dim within tile mt) ----
    if (tid == 0 && live) {
        tc_fence_after();
        constexpr uint32_t idO = idesc_f16_f32_mn_mn(128, NH);
        for (int mt = 0; mt < D / 128; ++mt)
            for (int kk = 0; kk < n16 / 16; ++kk)
                tc_mma_bf16(tbase + NH + NH * mt, smem_desc_sw128(sE + 2 * mt * lay.EREG + kk * 2048, lay.EREG, 1024),
                            smem_desc_sw128(sP + kk * 2048, 8192, 1024), idO, kk > 0);
        tc_commit(&bars[1]);
    }
    bool ok2 = true;
    if (live && tid == 0) ok2 = mbar_wait(&bars[1], 0, kWaitNs);
    ok2 = __syncthreads_and(ok2);
    if (!ok2 && tid == 0) set_status(a.status, LBCA_ERR_TIMEOUT);
    const bool have_o = live && ok2;
    griddep_launch_dependents();  // the next kernel on the stream may start its cache reads
    tc_fence_after();

    const int rope0 = D - a.rho;
    __nv_bfloat16* outp = static_cast<__nv_bfloat16*>(a.out) + ((size_t)b * a.Hq + (size_t)g * NH) * D;
    if (single) {
        // ---- the whole list was this CTA's: normalise and write straight from TMEM ----
        if (rank == 0) {
            if (tid < NH) {
                const float M = mh[tid];
                float dn = lloc[tid];
                if (a.sink && M != kNegInf) dn += ex2(sink_l2 - M);
                den[tid] = dn;
            }
            __syncthreads();
#pragma unroll 1
            for (int mt = 0; mt < D / 128; ++mt) {
                float o[16];
                if (have_o) {
                    tmem_ld16(tbase + lane_f + NH + NH * mt + 16 * hq, o);
                    tmem_wait_ld();
                }
                const int d = 128 * mt + 32 * quad + lane;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float dn = den[16 * hq + i];
                    float x = (have_o && dn > 0.f) ? o[i] / dn : 0.f;
                    const float y = __shfl_xor_sync(0xffffffffu, x, 1);  // pair partner (d ^ 1)
                    if (a.rho > 0 && d >= rope0) {
                        const float2 c = cs[(d - rope0) >> 1];
                        x = (d & 1) == 0 ? x * c.x + y * c.y : x * c.x - y * c.y;
                    }
                    outp[(size_t)(16 * hq + i) * D + d] = __float2bfloat16_rn(x);
                }
            }
        }
    } else {
        // ---- fp16 O^T slices to their owners, with this CTA's sums ----
        uint8_t* stage = smem + lay.OFF_E;  // [owner][NH/4][SW][4] fp16
#pragma unroll 1
        for (int mt = 0; mt < D / 128; ++mt) {
            float o[16];
            if (have_o) {
                tmem_ld16(tbase + lane_f + NH + NH * mt + 16 * hq, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) o[i] = 0.f;
            }
            const int d = 128 * mt + 32 * quad + lane;
            const int owner = d / SW, dd = d - owner * SW;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int h4 = 4 * hq + j;
                uint2 w2;
                w2.x = pack_f16x2(o[4 * j + 0], o[4 * j + 1]);
                w2.y = pack_f16x2(o[4 * j + 2], o[4 * j + 3]);
                *reinterpret_cast<uint2*>(stage + (size_t)owner * lay.SLICE + ((size_t)h4 * SW + dd) * 8) = w2;
            }
        }
        fence_async_smem();
        __syncthreads();
        if (tid < CS) {
            const uint32_t rb = peer_addr(bar_r, tid);
            bulk_to_peer(peer_addr(sQ + (uint32_t)rank * lay.SLICE, tid), smem_addr(stage) + tid * lay.SLICE,
                         lay.SLICE, rb);
            const uint32_t lo = smem_addr(smem + lay.OFF_LRECV) + (uint32_t)rank * NH * 4u;
            bulk_to_peer(peer_addr(lo, tid), smem_addr(lloc), NH * 4u, rb);
            bulk_commit();
        }
        // ---- owner: add the CS slices, normalise, rotate back, write ----
        const bool ok3 = __syncthreads_and(mbar_wait(&bars[3], 0, kWaitNs));
        if (!ok3 && tid == 0) set_status(a.status, LBCA_ERR_TIMEOUT);
        if (tid < NH) {
            const float M = mh[tid];
            float dn = 0.f;
            for (int r = 0; r < CS; ++r) dn += lrecv[r * NH + tid];
            if (a.sink && M != kNegInf) dn += ex2(sink_l2 - M);
            den[tid] = dn;
        }
        __syncthreads();
        const uint8_t* recv = smem + lay.OFF_Q;  // [src][NH/4][SW][4] fp16
        for (int u = tid; u < SW * (NH / 4); u += kThreads) {  // whole warps: SW * 16 is a multiple of 32
            const int h4 = u / SW, dd = u - h4 * SW;
            const int d = rank * SW + dd;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            if (ok3 && d < D) {
                for (int r = 0; r < CS; ++r) {
                    const uint2 w2 = *reinterpret_cast<const uint2*>(recv + (size_t)r * lay.SLICE +
                                                                     ((size_t)h4 * SW + dd) * 8);
                    const float2 p0 = unpack_f16x2(w2.x), p1 = unpack_f16x2(w2.y);
                    acc[0] += p0.x; acc[1] += p0.y; acc[2] += p1.x; acc[3] += p1.y;
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float dn = den[4 * h4 + j];
                float x = dn > 0.f ? acc[j] / dn : 0.f;
                const float y = __shfl_xor_sync(0xffffffffu, x, 1);  // pair partner (d ^ 1)
                if (a.rho > 0 && d >= rope0 && d < D) {
                    const float2 c = cs[(d - rope0) >> 1];
                    x = (d & 1) == 0 ? x * c.x + y * c.y : x * c.x - y * c.y;
                }
                if (d < D) outp[(size_t)(4 * h4 + j) * D + d] = __float2bfloat16_rn(x);
            }
        }
        if (tid < CS) bulk_wait_read_all();  // the staging is read out before this CTA exits
    }
    if (q_sender) bulk_wait_read_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

// How many CS-CTA clusters of this kernel fit on the device at once with `smem`
// bytes of shared memory per CTA (0: none).  Cached per cluster size.
template <int D>
int max_active_clusters(int cs, uint32_t smem) {
    auto fn = decode_mqa_tc_kernel<D>;
    static bool attr[64] = {};  // per device
    const int dev_ = current_device();
    if (dev_ < 0 || !attr[dev_]) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess ||
            cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        if (dev_ >= 0) attr[dev_] = true;
    }
    static uint32_t key[kMaxCS + 1];
    static int val[kMaxCS + 1];
    if (key[cs] == smem) return val[cs];
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(cs, 1, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int nclu = 0;
    if (cudaOccupancyMaxActiveClusters(&nclu, fn, &cfg) != cudaSuccess) {
        cudaGetLastError();
        nclu = 0;
    }
    key[cs] = smem;
    val[cs] = nclu;
    return nclu;
}

template <int D>
cudaError_t launch_d(const DecodeArgs& a, cudaStream_t s) {
    auto fn = decode_mqa_tc_kernel<D>;
    const MqaLayout lay(D, a.chunk, a.tc_cs);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.tc_cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(a.tc_cs, a.G, a.B);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = lay.SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = (a.pdl && !a.sel) ? 2 : 1;  // a selection comes from the preceding kernel: no early start
    return cudaLaunchKernelEx(&cfg, fn, a);
}

}  // namespace

namespace {
// Entry rows per CTA for cs CTAs per cluster over at most max_vis visible entries.
int rows_for(long long max_vis, int cs) {
    return std::max<int>(16, (int)(((max_vis + cs - 1) / cs + 15) / 16 * 16));
}
long long max_visible(int m, int w, int max_ctx) {
    const long long P = max_ctx - w > 0 ? (long long)(max_ctx - w) / m : 0;
    return std::min<long long>(max_ctx, P + w + m - 1);
}
}  // namespace

bool mqa_tc_shape_ok(int dtype, int B, int Hq, int G, int D, int m, int w, int shared, int max_ctx) {
    if (dtype != LBCA_BF16 || !shared || G < 1 || Hq != NH * G || (D != 256 && D != 512)) return false;
    if (B < 1 || max_ctx < 1) return false;
    const long long max_vis = max_visible(m, w, max_ctx);
    for (int cs = (int)std::max<long long>(1, (max_vis + 127) / 128); cs <= kMaxCS; ++cs)
        if (MqaLayout(D, rows_for(max_vis, cs), cs).SMEM <= 227u * 1024u) return true;
    return false;
}

MqaTcPlan plan_decode_mqa_tc(int dtype, int B, int Hq, int G, int D, int m, int w, int shared, int max_ctx) {
    if (!mqa_tc_shape_ok(dtype, B, Hq, G, D, m, w, shared, max_ctx)) return MqaTcPlan{0, 0};
    return plan_decode_mqa_tc_vis(dtype, B, Hq, G, D, shared, max_visible(m, w, max_ctx));
}

MqaTcPlan plan_decode_mqa_tc_vis(int dtype, int B, int Hq, int G, int D, int shared, long long max_vis) {
    MqaTcPlan p{0, 0};
    if (dtype != LBCA_BF16 || !shared || G < 1 || Hq != NH * G || (D != 256 && D != 512)) return p;
    if (B < 1 || max_vis < 1) return p;
    const int cs_min = (int)std::max<long long>(1, (max_vis + 127) / 128);
    // fewest waves of clusters first, then the widest cluster (the most SMs streaming)
    const long long groups = (long long)B * G;
    long long best_waves = 0;
    for (int cs = kMaxCS; cs >= cs_min; --cs) {
        const int rows = rows_for(max_vis, cs);
        const MqaLayout lay(D, rows, cs);
        if (lay.SMEM > 227u * 1024u) continue;
        const int act = D == 512 ? max_active_clusters<512>(cs, lay.SMEM) : max_active_clusters<256>(cs, lay.SMEM);
        if (act < 1) continue;
        const long long waves = (groups + act - 1) / act;
        if (p.cs == 0 || waves < best_waves) {
            p.cs = cs;
            p.rows = rows;
            best_waves = waves;
        }
    }
    return p;
}

cudaError_t launch_decode_mqa_tc(const DecodeArgs& a, cudaStream_t s) {
    if (a.B == 0) return cudaSuccess;
    if (a.D == 512) return launch_d<512>(a, s);
    if (a.D == 256) return launch_d<256>(a, s);
    return cudaErrorInvalidValue;
}

}  // namespace lbca
