// prefill_tc.cu -- causal block-compressed attention on the sm_100a tensor cores.
//
// Every query t attends, in one softmax, to the pooled entries j < P(t+1) and
// the raw tokens s in [P(t+1) m, t] (mSeek README, "How LBCA works", steps
// 4-5; HCA page, "What is implemented"), with RoPE on queries at t and on raw
// keys at s, pooled keys carrying RoPE at their block start (CSA page,
// "Deviations from paper").  This kernel serves the GQA form with bf16 I/O,
// head_dim 128 and no RMSNorm; other shapes use the CUDA-core kernel.
//
// B200 mapping (one CTA = 2 x 128 queries of one head, 384 threads):
//   warp 0     TMA producer: the two Q tiles once, then fp16 K and V tiles
//              of 64 entries (pooled tiles first, then the raw band) into a
//              four-stage ring, 128-byte swizzled, no multicast.
//   warps 1-2  MMA issuers, one per query tile q: S_q = Q_q K^T (tcgen05.mma
//              M=128 N=64, fp16 K-major operands from shared memory) into
//              q's TMEM S columns, and O_q += P V with P read from TMEM (one
//              of two P buffers) and fp16 V as an MN-major operand; completion
//              is signalled by tcgen05.commit on mbarriers.  S, P and O have
//              TMEM columns of their own, so S_q of the next tile is issued
//              as soon as the softmax has read the current one -- the tensor
//              core computes it while the exponentials of the current tile
//              run -- and P V of a tile runs behind.
//   warps 4-7, 8-11  softmax of query tiles 0 and 1: thread r owns query row r
//              and TMEM lane r.  It rotates its Q row in shared memory once,
//              then per tile loads its S row, releases S, applies the
//              causal-block / window mask, keeps an online max (rescaling O
//              in TMEM only when the max grows by more than 2^8), writes P in
//              fp16 into the free P buffer, and finally normalises its O row
//              (plus the sink) into shared memory, from where one thread
//              TMA-stores the tile.
// Raw keys arrive already rotated and, like the values, in fp16 (the pool pass
// writes them while it streams K and V, instead of every query tile converting
// them again); Q is
// rotated in shared memory from a per-position cos/sin table.  Rows past a tensor's valid extent
// are zero-filled by TMA, so masked products never meet garbage.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>

#include "kernels.h"
#include "tc.cuh"

namespace lbca {
namespace {

constexpr int BM = 128;     // query rows per softmax warpgroup (one M=128 MMA)
constexpr int NQ = 2;       // query tiles per CTA
constexpr int BN = 64;      // entries per K/V tile
constexpr int HD = 128;     // head dim
constexpr int NSTAGE = 4;   // K/V ring depth
constexpr uint32_t QREG = BM * 64 * 2;   // [128 rows][64 cols] 16-bit: one 128-byte swizzle span per row
constexpr uint32_t QTILE = 2 * QREG;     // [128][128]
constexpr uint32_t KREG = BN * 64 * 2;   // [64 rows][64 cols]
constexpr uint32_t KTILE = 2 * KREG;     // [64][128]
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + NQ * QTILE;
constexpr uint32_t OFF_V = OFF_K + NSTAGE * KTILE;
constexpr uint32_t OFF_BAR = OFF_V + NSTAGE * KTILE;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;  // + barriers, + alignment slack
// TMEM columns of query tile q, from 256 q: S [0, 64) f32, P buffers [64, 96) and
// [96, 128) (fp16 pairs: 64 entries in 32 columns), O [128, 256) f32.
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t T_S = 0, T_P = 64, T_O = 128;
constexpr int kThreads = 384;        // warps 0 producer, 1-2 MMA issuers, 3 idle, 4-7 / 8-11 softmax
constexpr uint64_t kWaitNs = 500ull * 1000 * 1000;

// barrier slots
constexpr int B_QFULL = 0;
constexpr int B_QROT = 1;                      // [NQ] softmax warpgroup q has rotated its Q rows
constexpr int B_KVFULL = B_QROT + NQ;          // [NSTAGE] the stage's K and V tiles have landed
constexpr int B_KVEMPTY = B_KVFULL + NSTAGE;   // [NSTAGE] both issuers are done with the stage
constexpr int B_SFULL = B_KVEMPTY + NSTAGE;    // [NQ] S_q computed
constexpr int B_SFREE = B_SFULL + NQ;          // [NQ] S_q read by the softmax
constexpr int B_PFULL = B_SFREE + NQ;          // [NQ] P_q written
constexpr int B_PVDONE = B_PFULL + NQ;         // [NQ][2] P V from P buffer b of query tile q done
constexpr int B_COUNT = B_PVDONE + 2 * NQ;

struct TcArgs {
    CUtensorMap tq;   // q [B, T, Hq, D] bf16          dims (D, Hq, T, B)
    CUtensorMap tpk;  // pooled keys fp16 [B, G, NB, D] dims (D, NB, G, B)
    CUtensorMap tpv;  // pooled values fp16
    CUtensorMap trk;  // finalised raw keys fp16 [B, T, G, D] dims (D, G, T, B)
    CUtensorMap trv;  // raw values fp16
    CUtensorMap to;   // out [B, T, Hq, D] bf16       dims (D, Hq, T, B)
    const float2* tab;  // [rho/2][T] cos/sin
    const float* sink;
    void* out;          // [B, T, Hq, D] bf16
    int32_t* status;
    int T, Hq, G, m, w, rho, n_ctiles;
    float scale;
};

__device__ __forceinline__ bool wait_or_fail(uint64_t* bar, uint32_t parity, int* fail, int32_t* status) {
    if (*reinterpret_cast<volatile int*>(fail)) return false;
    if (mbar_wait(bar, parity, kWaitNs)) return true;
    *reinterpret_cast<volatile int*>(fail) = 1;
    set_status(status, LBCA_ERR_TIMEOUT);
    return false;
}
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* fail, int32_t* status) {
    return __all_sync(0xffffffffu, wait_or_fail(bar, parity, fail, status));
}

// 2^x for a pair of values on the FMA pipe (packed f32x2), after Cody and
// Waite's range reduction: x = n + f with n = rint(x) and f in [-1/2, 1/2]; 2^f
// from a degree-3 polynomial (a weighted least-squares fit of 2^f on that
// interval, relative error below 7.5e-5, under half an fp16 ulp, the precision
// P is kept in); 2^n added to the exponent field.  Inputs below -125 (masked
// scores are -inf) give 2^-125, which is 0 in fp16; inputs are at most 8 here
// (the lazy rescale bounds them).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
    constexpr float kShift = 12582912.0f;  // 1.5 * 2^23: rint(x) lands in the low mantissa bits
    x.x = fmaxf(x.x, -125.0f);
    x.y = fmaxf(x.y, -125.0f);
    const float2 t = fadd2(x, make_float2(kShift, kShift));
    const float2 n = fadd2(t, make_float2(-kShift, -kShift));
    const float2 f = ffma2(n, make_float2(-1.0f, -1.0f), x);  // x - n, exact
    float2 p = ffma2(make_float2(0.0551716648f, 0.0551716648f), f, make_float2(0.2426111251f, 0.2426111251f));
    p = ffma2(p, f, make_float2(0.6932609677f, 0.6932609677f));
    p = ffma2(p, f, make_float2(0.9999280572f, 0.9999280572f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// The K/V tiles of a CTA run over the pooled entries [0, npt BN) and then the
// raw band [s_lo, t_last]; query tile q needs only a prefix of the pooled
// tiles and a sub-range of the raw tiles.  Tiles no row of q can see are not
// multiplied for q at all.
struct Need {
    int np;      // pooled tiles [0, np)
    int r0, r1;  // raw tiles [npt + r0, npt + r1)
    __device__ bool operator()(int i, int npt) const {
        return i < npt ? i < np : (i - npt >= r0 && i - npt < r1);
    }
};
__device__ __forceinline__ Need need_of(const TcArgs& a, int q, int t0, int s_lo, int nrt) {
    Need n{0, 0, 0};
    const int tf = t0 + q * BM;
    if (tf >= a.T) return n;
    const int tl = min(tf + BM, a.T) - 1;
    n.np = (visible_blocks(tl + 1, a.m, a.w) + BN - 1) / BN;
    const int lo = visible_blocks(tf + 1, a.m, a.w) * a.m;  // >= s_lo
    n.r0 = (lo - s_lo) / BN;
    n.r1 = min(nrt, tl >= s_lo ? (tl - s_lo) / BN + 1 : 0);
    n.r1 = max(n.r1, n.r0);
    return n;
}

__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ TcArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint32_t* tmem_sh = reinterpret_cast<uint32_t*>(bars + B_COUNT);
    int* fail = reinterpret_cast<int*>(tmem_sh + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x, ct = a.n_ctiles - 1 - (int)blockIdx.y, b = blockIdx.z;  // heavy tiles first
    const int g = h / (a.Hq / a.G);
    const int t0 = ct * NQ * BM;
    const int t_last = min(t0 + NQ * BM, a.T) - 1;
    const int Pmax = visible_blocks(t_last + 1, a.m, a.w);
    const int s_lo = visible_blocks(t0 + 1, a.m, a.w) * a.m;
    const int npt = (Pmax + BN - 1) / BN;
    const int nrt = (t_last - s_lo + 1 + BN - 1) / BN;
    const int ntile = npt + nrt;

    if (threadIdx.x == 0) {
        for (int i = 0; i < B_COUNT; ++i) {
            const bool softmax_arrivals = (i >= B_QROT && i < B_QROT + NQ) || (i >= B_SFREE && i < B_SFREE + NQ) ||
                                          (i >= B_PFULL && i < B_PFULL + NQ);
            const bool both_issuers = i >= B_KVEMPTY && i < B_KVEMPTY + NSTAGE;
            mbar_init(&bars[i], softmax_arrivals ? 128u : both_issuers ? (uint32_t)NQ : 1u);
        }
        *fail = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(tmem_sh, TMEM_COLS);
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_sh;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(&bars[B_QFULL], NQ * QTILE);
            for (int q = 0; q < NQ; ++q)
                for (int rg = 0; rg < 2; ++rg)
                    tma_load_4d(smem + OFF_Q + q * QTILE + rg * QREG, &a.tq, 64 * rg, h, t0 + q * BM, b,
                                &bars[B_QFULL]);
            int issued = 0;
            for (int i = 0; i < ntile; ++i) {
                const int s = i % NSTAGE;
                if (i >= NSTAGE && !wait_or_fail(&bars[B_KVEMPTY + s], ((i / NSTAGE) - 1) & 1, fail, a.status))
                    break;
                uint8_t* kd = smem + OFF_K + s * KTILE;
                uint8_t* vd = smem + OFF_V + s * KTILE;
                mbar_arrive_expect_tx(&bars[B_KVFULL + s], 2 * KTILE);
                if (i < npt) {
                    const int j0 = i * BN;
                    for (int rg = 0; rg < 2; ++rg) tma_load_4d(kd + rg * KREG, &a.tpk, 64 * rg, j0, g, b, &bars[B_KVFULL + s]);
                    for (int rg = 0; rg < 2; ++rg) tma_load_4d(vd + rg * KREG, &a.tpv, 64 * rg, j0, g, b, &bars[B_KVFULL + s]);
                } else {
                    const int s0 = s_lo + (i - npt) * BN;
                    for (int rg = 0; rg < 2; ++rg) tma_load_4d(kd + rg * KREG, &a.trk, 64 * rg, g, s0, b, &bars[B_KVFULL + s]);
                    for (int rg = 0; rg < 2; ++rg) tma_load_4d(vd + rg * KREG, &a.trv, 64 * rg, g, s0, b, &bars[B_KVFULL + s]);
                }
                issued = i + 1;
            }
            // drain: never leave copies in flight into shared memory (bounded)
            for (int i = max(0, issued - NSTAGE); i < issued; ++i) {
                mbar_wait(&bars[B_KVFULL + i % NSTAGE], (i / NSTAGE) & 1, kWaitNs);
            }
            mbar_wait(&bars[B_QFULL], 0, kWaitNs);
        }
    } else if (warp == 1 || warp == 2) {
        // ------------------------------------------- MMA issuers, one per query tile
        // For each tile i this query tile needs: S(i) once K(i) has landed and
        // the softmax has read S of the previous tile, then P V of the previous
        // tile (so the tensor core computes S(i) while the softmax of the
        // previous tile runs).  A stage is released (KVEMPTY, two issuers) after
        // its P V; a tile no row of q can see is released once its data has
        // landed.  A pending P V is issued early when the next wait would need
        // the stage it holds.
        const int q = warp - 1;
        if (lane == 0) {
            const uint32_t idS = idesc_f16_f32(BM, BN, false);
            const uint32_t idP = idesc_f16_f32(BM, HD, true);
            const uint32_t tq = tbase + 256 * q;
            // descriptors of each operand's first 16-column step; later steps add their
            // byte offset >> 4 to the start-address field (no carry: shared addresses < 2^18)
            const uint64_t dq = smem_desc_sw128(smem_addr(smem + OFF_Q + q * QTILE), 16, 1024);
            const uint64_t dk = smem_desc_sw128(smem_addr(smem + OFF_K), 16, 1024);
            const uint64_t dv = smem_desc_sw128(smem_addr(smem + OFF_V), KREG, 1024);
            const Need nd = need_of(a, q, t0, s_lo, nrt);
            bool ok = wait_or_fail(&bars[B_QROT + q], 0, fail, a.status);
            int k = 0;      // needed tiles whose S has been issued
            int prev = -1;  // tile whose P V is still to be issued (the (k-1)-th needed one)
            auto issue_pv = [&](int i, int kk) {  // P V of tile i, the kk-th needed tile of q
                ok = wait_or_fail(&bars[B_PFULL + q], kk & 1, fail, a.status);  // (its data landed before S(i))
                if (!ok) return;
                const uint64_t dvs = dv + (((i % NSTAGE) * KTILE) >> 4);
                tc_fence_after();
#pragma unroll
                for (int e = 0; e < BN / 16; ++e)  // A = P (16 entries = 8 fp16-pair columns)
                    tc_mma_ts(tq + T_O, tq + T_P + 32 * (kk & 1) + 8 * e, dvs + ((e * 2048) >> 4), idP,
                              (kk > 0 || e > 0) ? 1u : 0u);
                tc_commit(&bars[B_PVDONE + 2 * q + (kk & 1)]);
                tc_commit(&bars[B_KVEMPTY + i % NSTAGE]);
            };
            for (int i = 0; ok && i < ntile; ++i) {
                if (prev >= 0 && prev <= i - NSTAGE) {  // tile i reuses prev's stage
                    issue_pv(prev, k - 1);
                    prev = -1;
                    if (!ok) break;
                }
                if (!nd(i, npt)) {
                    ok = wait_or_fail(&bars[B_KVFULL + i % NSTAGE], (i / NSTAGE) & 1, fail, a.status);
                    if (ok) tc_commit(&bars[B_KVEMPTY + i % NSTAGE]);
                    continue;
                }
                ok = wait_or_fail(&bars[B_KVFULL + i % NSTAGE], (i / NSTAGE) & 1, fail, a.status);
                if (ok && k > 0) ok = wait_or_fail(&bars[B_SFREE + q], (k - 1) & 1, fail, a.status);
                if (!ok) break;
                const uint64_t dks = dk + (((i % NSTAGE) * KTILE) >> 4);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    tc_mma_bf16(tq + T_S, dq + (((kk >> 2) * QREG + (kk & 3) * 32) >> 4),
                                dks + (((kk >> 2) * KREG + (kk & 3) * 32) >> 4), idS, kk > 0);
                tc_commit(&bars[B_SFULL + q]);
                if (prev >= 0) issue_pv(prev, k - 1);
                prev = i;
                ++k;
            }
            if (ok && prev >= 0) issue_pv(prev, k - 1);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------- softmax
        const int q = (warp - 4) >> 2;           // query tile of this warpgroup
        const int r = threadIdx.x - 128 - 128 * q;
        const int t = t0 + q * BM + r;
        const bool valid = t < a.T;
        const int Pq = visible_blocks(t + 1, a.m, a.w);
        const int lo = Pq * a.m;
        const uint32_t lane_f = (uint32_t)(32 * (warp & 3)) << 16;
        const int half = a.rho / 2;
        const uint32_t tS = tbase + 256 * q + lane_f + T_S;
        const uint32_t tP = tbase + 256 * q + lane_f + T_P;
        const uint32_t tO = tbase + 256 * q + lane_f + T_O;
        uint8_t* sQ = smem + OFF_Q + q * QTILE;

        // this query row's cos/sin, fetched in one batch while Q lands
        float2 cs_row[HD / 2];
        {
            const int base = HD / 2 - half;  // pairs below `base` are not rotated
            const float2* tab = a.tab + (valid ? t : 0);  // pair-major: a warp's 32 rows are contiguous
#pragma unroll
            for (int k = 0; k < HD / 2; ++k)
                cs_row[k] = (valid && k >= base) ? __ldg(tab + (size_t)(k - base) * a.T) : make_float2(1.f, 0.f);
        }
        bool ok = warp_wait(&bars[B_QFULL], 0, fail, a.status);
        if (ok) {  // this query row, in place: bf16 -> f32, RoPE at t, -> fp16 (QK^T runs in fp16)
            bool ovf = false;  // a value beyond the fp16 range would become inf
#pragma unroll
            for (int c8 = 0; c8 < HD / 8; ++c8) {
                uint4* p = reinterpret_cast<uint4*>(sQ + sw128_off(r, 8 * c8, QREG));
                uint4 u = *p;
                uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float x = __uint_as_float(wv[e] << 16), y = __uint_as_float(wv[e] & 0xffff0000u);
                    rotate_pair(x, y, cs_row[4 * c8 + e]);
                    ovf |= fabsf(x) > 65504.f || fabsf(y) > 65504.f;
                    wv[e] = pack_f16x2(x, y);
                }
                *p = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
            if (ovf) set_status(a.status, LBCA_ERR_UNSUPPORTED);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&bars[B_QROT + q]);

        const float sc = a.scale * kLog2e;  // scores enter the exponent as s * sc (log2 units)
        float m_ref = kNegInf, l = 0.f;     // running max (unscaled score units) and sum
        const Need nd = need_of(a, q, t0, s_lo, nrt);
        int k = 0;                          // tiles of this query tile so far
        for (int i = 0; ok && i < ntile; ++i) {
            if (!nd(i, npt)) continue;      // uniform over the warpgroup
            const bool pooled = i < npt;
            const int base = pooled ? i * BN : s_lo + (i - npt) * BN;
            ok = warp_wait(&bars[B_SFULL + q], k & 1, fail, a.status);
            if (!ok) break;
            tc_fence_after();
            float s[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                float v[32];
                tmem_ld32(tS + 32 * c, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) s[32 * c + e] = v[e];
            }
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars[B_SFREE + q]);  // S may be overwritten by the next tile's S

            // visible columns of this row in this tile: [c_lo, c_hi)
            int c_lo, c_hi;
            if (pooled) { c_lo = 0; c_hi = min(BN, Pq - base); }
            else { c_lo = max(0, lo - base); c_hi = min(BN, t - base + 1); }
            if (!valid) c_hi = 0;
            c_hi = max(c_hi, c_lo);  // an empty range masks every column
            if (__any_sync(0xffffffffu, c_lo > 0 || c_hi < BN)) {
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if ((unsigned)(c - c_lo) >= (unsigned)(c_hi - c_lo)) s[c] = kNegInf;
            }
            float mxv[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
#pragma unroll
            for (int c = 0; c < BN / 2; ++c) mxv[c & 3] = fmax3(mxv[c & 3], s[2 * c], s[2 * c + 1]);
            const float mx = fmax3(fmaxf(mxv[0], mxv[1]), mxv[2], mxv[3]);
            // lazy rescale: only when the row max grows by more than 2^8 in probability
            float alpha = 1.f;
            bool rescale = false;
            if (mx * sc > m_ref * sc + 8.f) {  // also the first visible score (m_ref = -inf)
                alpha = m_ref == kNegInf ? 0.f : ex2((m_ref - mx) * sc);
                rescale = m_ref != kNegInf;
                m_ref = mx;
            }
            const float mneg = m_ref == kNegInf ? 0.f : -m_ref * sc;
            if (__any_sync(0xffffffffu, rescale)) {
                // O must be quiet: every P V issued so far (up to tile k-1) has completed
                if (k > 0) ok = warp_wait(&bars[B_PVDONE + 2 * q + ((k - 1) & 1)], ((k - 1) >> 1) & 1, fail, a.status);
                if (!ok) break;
                tc_fence_after();
                const float f = rescale ? alpha : 1.f;
#pragma unroll 1
                for (int c = 0; c < HD / 32; ++c) {
                    float v[32];
                    tmem_ld32(tO + 32 * c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] *= f;
                    tmem_st32(tO + 32 * c, v);
                }
            }
            // P buffer k & 1 is free once the P V of tile k-2 has read it
            if (k >= 2) ok = warp_wait(&bars[B_PVDONE + 2 * q + (k & 1)], ((k >> 1) - 1) & 1, fail, a.status);
            if (!ok) break;
            // exponentials in pairs: pairs 1, 4 and 6 of every 8 on the FMA pipe
            // (packed polynomial), the rest on the SFU, which 3/8 relieves enough
            // for the two warps sharing each SFU to keep pace with the FMA pipe
            float2 ps[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            float pk[32];
            const float2 sc2 = make_float2(sc, sc), mn2 = make_float2(mneg, mneg);
#pragma unroll
            for (int e = 0; e < BN / 2; ++e) {
                const float2 x = ffma2(make_float2(s[2 * e], s[2 * e + 1]), sc2, mn2);
                float2 p;
                if ((0x52u >> (e & 7)) & 1u) {
                    p = exp2_fma2(x);
                } else {
                    p.x = ex2(x.x);
                    p.y = ex2(x.y);
                }
                ps[e & 1] = fadd2(ps[e & 1], p);
                pk[e] = __uint_as_float(pack_f16x2(p.x, p.y));
            }
            tc_fence_after();
            tmem_st32(tP + 32 * (k & 1), pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[B_PFULL + q]);
            l = l * alpha + ((ps[0].x + ps[0].y) + (ps[1].x + ps[1].y));
            ++k;
        }
        // ---- epilogue: normalise the O row into this query tile's shared memory
        // (free: the last S MMA that read Q is complete), then TMA-store the tile
        if (ok && k > 0) ok = warp_wait(&bars[B_PVDONE + 2 * q + ((k - 1) & 1)], ((k - 1) >> 1) & 1, fail, a.status);
        tc_fence_after();
        float den = l;
        if (a.sink) den += m_ref == kNegInf ? 1.f : ex2(a.sink[h] * kLog2e - m_ref * sc);
        const float inv = den > 0.f ? 1.f / den : 0.f;
        const bool have_o = ok && k > 0;  // warp-uniform
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
            float v[32];
            if (have_o) {  // every lane loads (warp-collective)
                tmem_ld32(tO + 32 * c, v);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int k = 0; k < 32; ++k) v[k] = 0.f;
            }
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                uint4 u;
                u.x = pack_bf16x2(v[8 * c8 + 0] * inv, v[8 * c8 + 1] * inv);
                u.y = pack_bf16x2(v[8 * c8 + 2] * inv, v[8 * c8 + 3] * inv);
                u.z = pack_bf16x2(v[8 * c8 + 4] * inv, v[8 * c8 + 5] * inv);
                u.w = pack_bf16x2(v[8 * c8 + 6] * inv, v[8 * c8 + 7] * inv);
                *reinterpret_cast<uint4*>(sQ + sw128_off(r, 32 * c + 8 * c8, QREG)) = u;
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        named_barrier(1 + q, 128);
        if (r == 0) {
            tma_store_4d(&a.to, sQ, 0, h, t0 + q * BM, b);
            tma_store_4d(&a.to, sQ + QREG, 64, h, t0 + q * BM, b);
            tma_store_commit_and_wait_read();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

// cos/sin of every (pair, position) the queries and raw keys need, pair-major
// ([half][T]) so that consecutive positions of one pair are contiguous.
__global__ void rope_table_kernel(float2* tab, int T, int half, double step) {
    const int64_t n = (int64_t)T * half;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        tab[i] = rope_cs(i % T, (int)(i / T), step);
}

// Finalised raw keys (RoPE at s applied once) and raw values of tokens
// [s_begin, T), both widened to fp16, the operand type of the tensor-core MMAs;
// same [B, T, G, D] layout.  (The pool pass writes those of complete blocks.)
__global__ void finalise_kv_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                                   __half* __restrict__ ko, __half* __restrict__ vo, const float2* __restrict__ tab,
                                   int64_t n_vec, int G, int T, int s_begin, int rho, int32_t* status) {
    bool ovf = false;  // a value beyond the fp16 range would become inf
    const int64_t per_b = (int64_t)(T - s_begin) * G * (HD / 8);  // vectors of one sequence's tail
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n_vec; j += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = j / per_b;
        const int64_t i = (b * T + s_begin) * G * (HD / 8) + j % per_b;  // vector index in [B, T, G, D / 8]
        const int d0 = (int)(i % (HD / 8)) * 8;
        const int64_t row = i / (HD / 8);            // (b, s, g)
        const int s = (int)((row / G) % T);
        float x[8], y[8];
        ld16(k + i * 8, x);
        ld16(v + i * 8, y);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const int d = d0 + e;
            if (d >= HD - rho) rotate_pair(x[e], x[e + 1], tab[(size_t)((d - (HD - rho)) >> 1) * T + s]);
        }
        st16_f16_checked(ko + i * 8, x, ovf);
        st16_f16_checked(vo + i * 8, y, ovf);
    }
    if (ovf) set_status(status, LBCA_ERR_UNSUPPORTED);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 4-D bf16 map with a box of (64, b1, b2, 1) and 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, const uint64_t dims[4], const uint64_t strides_bytes[3],
              uint32_t box1, uint32_t box2, bool f16 = false) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t box[4] = {64, box1, box2, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                    const_cast<void*>(base), dims, strides_bytes, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

bool prefill_tc_supported(int dtype, int D, int rmsnorm, int shared) {
    return dtype == LBCA_BF16 && D == HD && !rmsnorm && !shared;
}

// scratch: [fp16 raw keys][fp16 raw values][cos/sin table][fp16 pooled keys][fp16 pooled values]
static size_t a256(size_t x) { return (x + 255) / 256 * 256; }
size_t prefill_tc_pooled_f16_offset(int B, int T, int G, int rho) {
    const size_t raw = a256((size_t)B * T * G * HD * 2);
    const size_t tab = a256((size_t)T * std::max(rho / 2, 1) * sizeof(float2));
    return 2 * raw + tab;
}
size_t prefill_tc_pooled_v_f16_offset(int B, int T, int G, int rho, int m) {
    return prefill_tc_pooled_f16_offset(B, T, G, rho) + a256((size_t)B * G * (T / m) * HD * 2);
}
size_t prefill_tc_scratch_bytes(int B, int T, int G, int rho, int m) {
    return prefill_tc_pooled_v_f16_offset(B, T, G, rho, m) + a256((size_t)B * G * (T / m) * HD * 2);
}

PrefillRawF16 prefill_tc_raw_f16(const PrefillArgs& p, void* scratch) {
    const size_t raw_bytes = a256((size_t)p.B * p.T * p.G * HD * 2);
    PrefillRawF16 r;
    r.keys = scratch;
    r.vals = static_cast<char*>(scratch) + raw_bytes;
    r.tab = reinterpret_cast<const float2*>(static_cast<char*>(scratch) + 2 * raw_bytes);
    return r;
}

cudaError_t launch_prefill_tc_table(const PrefillArgs& p, void* scratch, cudaStream_t s) {
    const int half = p.rho / 2;
    if (p.B == 0 || p.T == 0 || half == 0) return cudaSuccess;
    float2* tab = const_cast<float2*>(prefill_tc_raw_f16(p, scratch).tab);
    const int64_t n = (int64_t)p.T * half;
    rope_table_kernel<<<(int)std::min<int64_t>((n + 255) / 256, 148 * 16), 256, 0, s>>>(tab, p.T, half, p.rope_step);
    return cudaGetLastError();
}

cudaError_t launch_prefill_tc(const PrefillArgs& p, void* scratch, int32_t* status, cudaStream_t s) {
    if (p.B == 0 || p.T == 0) return cudaSuccess;
    const int G = p.G, T = p.T, B = p.B, Hq = p.Hq;
    const PrefillRawF16 raw = prefill_tc_raw_f16(p, scratch);
    __half* keys = static_cast<__half*>(raw.keys);
    __half* vals = static_cast<__half*>(raw.vals);
    const float2* tab = raw.tab;
    const void* pooled_k16 = static_cast<char*>(scratch) + prefill_tc_pooled_f16_offset(B, T, G, p.rho);
    const void* pooled_v16 = static_cast<char*>(scratch) + prefill_tc_pooled_v_f16_offset(B, T, G, p.rho, p.m);
    const int s_begin = T / p.m * p.m;  // tokens of complete blocks came from the pool pass
    if (s_begin < T) {
        const int64_t nv = (int64_t)B * (T - s_begin) * G * (HD / 8);
        finalise_kv_kernel<<<(int)std::min<int64_t>((nv + 255) / 256, 148 * 32), 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(p.k), static_cast<const __nv_bfloat16*>(p.v), keys, vals, tab, nv, G, T,
            s_begin, p.rho, status);
    }
    TcArgs a;
    memset(&a, 0, sizeof(a));
    const uint64_t e = 2;
    {   // q [B, T, Hq, D]
        const uint64_t dims[4] = {HD, (uint64_t)Hq, (uint64_t)T, (uint64_t)B};
        const uint64_t str[3] = {HD * e, (uint64_t)Hq * HD * e, (uint64_t)T * Hq * HD * e};
        if (!make_map(&a.tq, p.q, dims, str, 1, BM)) return cudaErrorInvalidValue;  // box 64 x 1 x 128
        if (!make_map(&a.to, p.out, dims, str, 1, BM)) return cudaErrorInvalidValue;
    }
    const int NB = T / p.m;
    const uint64_t ps = (uint64_t)std::max(p.pool_stride, 1);
    {   // pooled [B, G, stride, D], valid rows NB
        const uint64_t dims[4] = {HD, (uint64_t)std::max(NB, 1), (uint64_t)G, (uint64_t)B};
        const uint64_t str[3] = {HD * e, ps * HD * e, (uint64_t)G * ps * HD * e};
        // fp16 pooled keys and values in the scratch, [B, G, NB, D]
        const uint64_t nb = (uint64_t)std::max(NB, 1);
        const uint64_t str16[3] = {HD * e, nb * HD * e, (uint64_t)G * nb * HD * e};
        if (!make_map(&a.tpk, pooled_k16, dims, str16, BN, 1, true)) return cudaErrorInvalidValue;
        if (!make_map(&a.tpv, pooled_v16, dims, str16, BN, 1, true)) return cudaErrorInvalidValue;
        (void)str;
    }
    {   // raw [B, T, G, D]
        const uint64_t dims[4] = {HD, (uint64_t)G, (uint64_t)T, (uint64_t)B};
        const uint64_t str[3] = {HD * e, (uint64_t)G * HD * e, (uint64_t)T * G * HD * e};
        if (!make_map(&a.trk, keys, dims, str, 1, BN, true)) return cudaErrorInvalidValue;
        if (!make_map(&a.trv, vals, dims, str, 1, BN, true)) return cudaErrorInvalidValue;
    }
    a.tab = tab;
    a.sink = p.sink;
    a.out = p.out;
    a.status = status;
    a.T = T; a.Hq = Hq; a.G = G; a.m = p.m; a.w = p.w; a.rho = p.rho;
    a.n_ctiles = (T + NQ * BM - 1) / (NQ * BM);
    a.scale = p.scale;
    static bool attr_set[64] = {};  // per device
    const int dev_ = current_device();
    if (dev_ < 0 || !attr_set[dev_]) {
        cudaError_t err = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)SMEM_BYTES);
        if (err != cudaSuccess) return err;
        if (dev_ >= 0) attr_set[dev_] = true;
    }
    dim3 grid(Hq, a.n_ctiles, B);
    prefill_tc_kernel<<<grid, kThreads, SMEM_BYTES, s>>>(a);
    return cudaGetLastError();
}

}  // namespace lbca
