// prefill_tc.cu -- causal block-compressed attention on the sm_100a tensor cores.
//
// Every query t attends, in one softmax, to the pooled entries j < P(t+1) and
// the raw tokens s in [P(t+1) m, t] (mSeek README, "How LBCA works", steps
// 4-5; HCA page, "What is implemented"), with RoPE on queries at t and on raw
// keys at s, pooled keys carrying RoPE at their block start (CSA page,
// "Deviations from paper").  This kernel serves the GQA form with bf16 I/O,
// head_dim 128 and no RMSNorm; other shapes use the CUDA-core kernel.
//
// B200 mapping (one CTA = 128 queries of one head, 256 threads):
//   warp 0     TMA producer: the Q tile once, then K and V tiles of 128
//              entries (pooled tiles first, then the raw band) into a
//              two-stage ring, 128-byte swizzled, no multicast.
//   warp 1     TMEM owner and MMA issuer: S = Q K^T (tcgen05.mma M=128 N=128,
//              K-major operands) into one of two TMEM S buffers, and
//              O += P V (fp16 P from shared memory, fp16 V as an MN-major operand) into
//              the TMEM O accumulator; completion is signalled by
//              tcgen05.commit on mbarriers.  S(i+1) is issued before PV(i) so
//              the tensor core works on the next tile while the softmax runs.
//   warps 2-3  convert each V tile in place from bf16 to fp16 once it lands.
//   warps 4-7  softmax: thread r owns query row r and TMEM lane r.  It rotates
//              its Q row in shared memory once, then per tile loads its S row,
//              applies the causal-block / window mask, keeps an online max
//              (rescaling O in TMEM only when the max grows by more than 2^8),
//              writes P in fp16 into the swizzled P tile, and finally
//              normalises its O row (plus the sink) and stores it.
// Raw keys arrive already rotated (a pre-pass writes the finalised keys once,
// instead of every query tile rotating them again); Q is rotated in shared
// memory from a per-position cos/sin table.  Rows past a tensor's valid extent
// are zero-filled by TMA, so masked products never meet garbage.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>

#include "kernels.h"
#include "tc.cuh"

namespace lbca {
namespace {

constexpr int BM = 128, BN = 128, HD = 128;
constexpr uint32_t REGION = 128 * 64 * 2;  // [128 rows][64 cols] bf16, one 128-byte swizzle span per row
constexpr uint32_t TILE = 2 * REGION;      // a [128][128] bf16 tile
constexpr uint32_t OFF_Q = 0, OFF_K = TILE, OFF_V = 3 * TILE, OFF_P = 5 * TILE, OFF_BAR = 6 * TILE;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;  // + barriers, + alignment slack
constexpr uint32_t TMEM_COLS = 512;                    // S0, S1, O (128 columns each)
constexpr uint64_t kWaitNs = 500ull * 1000 * 1000;

enum { B_QFULL, B_QROT, B_KFULL0, B_KFULL1, B_VFULL0, B_VFULL1, B_VCONV0, B_VCONV1, B_KVEMPTY0, B_KVEMPTY1,
       B_SFULL0, B_SFULL1, B_SFREE0, B_SFREE1, B_PFULL, B_ODONE, B_COUNT };

struct TcArgs {
    CUtensorMap tq;   // q [B, T, Hq, D]          dims (D, Hq, T, B)
    CUtensorMap tpk;  // pooled keys [B, G, *, D]  dims (D, NB, G, B)
    CUtensorMap tpv;  // pooled values
    CUtensorMap trk;  // finalised raw keys [B, T, G, D] dims (D, G, T, B)
    CUtensorMap trv;  // raw values
    const float2* tab;  // [T][rho/2] cos/sin
    const float* sink;
    void* out;          // [B, T, Hq, D] bf16
    int32_t* status;
    int T, Hq, G, m, w, rho, n_qtiles;
    float scale;
};

__device__ __forceinline__ bool wait_or_fail(uint64_t* bar, uint32_t parity, int* fail, int32_t* status) {
    if (*reinterpret_cast<volatile int*>(fail)) return false;
    if (mbar_wait(bar, parity, kWaitNs)) return true;
    *reinterpret_cast<volatile int*>(fail) = 1;
    set_status(status, LBCA_ERR_TIMEOUT);
    return false;
}

__global__ void __launch_bounds__(256, 1) prefill_tc_kernel(const __grid_constant__ TcArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint32_t* tmem_sh = reinterpret_cast<uint32_t*>(bars + B_COUNT);
    int* fail = reinterpret_cast<int*>(tmem_sh + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x, qt = a.n_qtiles - 1 - (int)blockIdx.y, b = blockIdx.z;  // heavy tiles first
    const int g = h / (a.Hq / a.G);
    const int t0 = qt * BM;
    const int t_last = min(t0 + BM, a.T) - 1;
    const int Pmax = visible_blocks(t_last + 1, a.m, a.w);
    const int s_lo = visible_blocks(t0 + 1, a.m, a.w) * a.m;
    const int npt = (Pmax + BN - 1) / BN;
    const int nrt = (t_last - s_lo + 1 + BN - 1) / BN;
    const int ntile = npt + nrt;

    if (threadIdx.x == 0) {
        for (int i = 0; i < B_COUNT; ++i) {
            const bool softmax_arrivals = i == B_QROT || i == B_SFREE0 || i == B_SFREE1 || i == B_PFULL;
            const bool convert_arrivals = i == B_VCONV0 || i == B_VCONV1;
            mbar_init(&bars[i], softmax_arrivals ? 128u : convert_arrivals ? 64u : 1u);
        }
        *fail = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(tmem_sh, TMEM_COLS);
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_sh;
    const uint32_t tO = tbase + 256;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(&bars[B_QFULL], TILE);
            tma_load_4d(smem + OFF_Q, &a.tq, 0, h, t0, b, &bars[B_QFULL]);
            tma_load_4d(smem + OFF_Q + REGION, &a.tq, 64, h, t0, b, &bars[B_QFULL]);
            int issued = 0;
            for (int i = 0; i < ntile; ++i) {
                const int s = i & 1;
                if (i >= 2 && !wait_or_fail(&bars[B_KVEMPTY0 + s], ((i >> 1) - 1) & 1, fail, a.status)) break;
                uint8_t* kd = smem + OFF_K + s * TILE;
                uint8_t* vd = smem + OFF_V + s * TILE;
                mbar_arrive_expect_tx(&bars[B_KFULL0 + s], TILE);
                mbar_arrive_expect_tx(&bars[B_VFULL0 + s], TILE);
                if (i < npt) {
                    const int j0 = i * BN;
                    tma_load_4d(kd, &a.tpk, 0, j0, g, b, &bars[B_KFULL0 + s]);
                    tma_load_4d(kd + REGION, &a.tpk, 64, j0, g, b, &bars[B_KFULL0 + s]);
                    tma_load_4d(vd, &a.tpv, 0, j0, g, b, &bars[B_VFULL0 + s]);
                    tma_load_4d(vd + REGION, &a.tpv, 64, j0, g, b, &bars[B_VFULL0 + s]);
                } else {
                    const int s0 = s_lo + (i - npt) * BN;
                    tma_load_4d(kd, &a.trk, 0, g, s0, b, &bars[B_KFULL0 + s]);
                    tma_load_4d(kd + REGION, &a.trk, 64, g, s0, b, &bars[B_KFULL0 + s]);
                    tma_load_4d(vd, &a.trv, 0, g, s0, b, &bars[B_VFULL0 + s]);
                    tma_load_4d(vd + REGION, &a.trv, 64, g, s0, b, &bars[B_VFULL0 + s]);
                }
                issued = i + 1;
            }
            // drain: never leave copies in flight into shared memory (bounded)
            for (int i = max(0, issued - 2); i < issued; ++i) {
                mbar_wait(&bars[B_KFULL0 + (i & 1)], (i >> 1) & 1, kWaitNs);
                mbar_wait(&bars[B_VFULL0 + (i & 1)], (i >> 1) & 1, kWaitNs);
            }
            mbar_wait(&bars[B_QFULL], 0, kWaitNs);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idS = idesc_f16_f32(BM, BN, false);
            const uint32_t idP = idesc_f16_f32(BM, HD, true);
            const uint32_t sq = smem_addr(smem + OFF_Q), sp = smem_addr(smem + OFF_P);
            auto issue_s = [&](int i) {
                const int s = i & 1;
                const uint32_t sk = smem_addr(smem + OFF_K + s * TILE);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * REGION + (kk & 3) * 32;
                    tc_mma_bf16(tbase + 128 * s, smem_desc_sw128(sq + off, 16, 1024),
                                smem_desc_sw128(sk + off, 16, 1024), idS, kk > 0);
                }
                tc_commit(&bars[B_SFULL0 + s]);
            };
            bool ok = wait_or_fail(&bars[B_QROT], 0, fail, a.status);
            if (ok && ntile > 0) ok = wait_or_fail(&bars[B_KFULL0], 0, fail, a.status);
            if (ok && ntile > 0) issue_s(0);
            for (int i = 0; ok && i < ntile; ++i) {
                const int n = i + 1;
                if (n < ntile) {
                    ok = wait_or_fail(&bars[B_KFULL0 + (n & 1)], (n >> 1) & 1, fail, a.status);
                    if (ok && n >= 2) ok = wait_or_fail(&bars[B_SFREE0 + (n & 1)], ((n >> 1) - 1) & 1, fail, a.status);
                    if (!ok) break;
                    issue_s(n);
                }
                ok = wait_or_fail(&bars[B_PFULL], i & 1, fail, a.status) &&
                     wait_or_fail(&bars[B_VCONV0 + (i & 1)], (i >> 1) & 1, fail, a.status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sv = smem_addr(smem + OFF_V + (i & 1) * TILE);
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint32_t poff = (kk >> 2) * REGION + (kk & 3) * 32;
                    tc_mma_bf16(tO, smem_desc_sw128(sp + poff, 16, 1024),
                                smem_desc_sw128(sv + kk * 2048, REGION, 1024), idP, (i > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&bars[B_ODONE]);
                tc_commit(&bars[B_KVEMPTY0 + (i & 1)]);
            }
        }
    } else if (warp == 2 || warp == 3) {
        // ----------------------------------------- V tiles: bf16 -> fp16 in place
        // (P V runs in fp16: P in [0, 256] keeps 11 mantissa bits; bf16 values
        // widen exactly to fp16 in its normal range; element-wise, so the
        // swizzled layout is untouched)
        const int ct = threadIdx.x - 64;
        for (int i = 0; i < ntile; ++i) {
            const int s = i & 1;
            if (!__all_sync(0xffffffffu, wait_or_fail(&bars[B_VFULL0 + s], (i >> 1) & 1, fail, a.status))) break;
            uint4* vt = reinterpret_cast<uint4*>(smem + OFF_V + s * TILE);
            for (int q = ct; q < (int)(TILE / 16); q += 64) {
                uint4 u = vt[q];
                uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    wv[e] = pack_f16x2(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xffff0000u));
                vt[q] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(&bars[B_VCONV0 + s]);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------- softmax
        const int r = threadIdx.x - 128;
        const int t = t0 + r;
        const bool valid = t < a.T;
        const int Pq = visible_blocks(t + 1, a.m, a.w);
        const int lo = Pq * a.m;
        const uint32_t lane_f = (uint32_t)(32 * (warp - 4)) << 16;
        const int half = a.rho / 2;

        bool ok = __all_sync(0xffffffffu, wait_or_fail(&bars[B_QFULL], 0, fail, a.status));
        if (ok) {  // this query row, in place: bf16 -> f32, RoPE at t, -> fp16 (QK^T runs in fp16)
            const float2* tab = a.tab + (size_t)(valid ? t : 0) * half;
            for (int q = 0; q < HD / 8; ++q) {
                uint4* p = reinterpret_cast<uint4*>(smem + OFF_Q + sw128_off(r, 8 * q, REGION));
                uint4 u = *p;
                uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int d = 8 * q + 2 * e;
                    float x = __uint_as_float(wv[e] << 16), y = __uint_as_float(wv[e] & 0xffff0000u);
                    if (valid && d >= HD - a.rho) rotate_pair(x, y, tab[(d - (HD - a.rho)) >> 1]);
                    wv[e] = pack_f16x2(x, y);
                }
                *p = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&bars[B_QROT]);

        const float sc = a.scale * kLog2e;
        float m_ref = kNegInf, l = 0.f;
        for (int i = 0; ok && i < ntile; ++i) {
            const bool pooled = i < npt;
            const int base = pooled ? i * BN : s_lo + (i - npt) * BN;
            ok = __all_sync(0xffffffffu, wait_or_fail(&bars[B_SFULL0 + (i & 1)], (i >> 1) & 1, fail, a.status));
            if (!ok) break;
            tc_fence_after();
            float s[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                float v[32];
                tmem_ld32(tbase + 128 * (i & 1) + lane_f + 32 * c, v);
#pragma unroll
                for (int k = 0; k < 32; ++k) s[32 * c + k] = v[k];
            }
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars[B_SFREE0 + (i & 1)]);

            float mx = kNegInf;
#pragma unroll
            for (int c = 0; c < BN; ++c) {
                const int e = base + c;
                const bool vis = valid && (pooled ? e < Pq : (e >= lo && e <= t));
                s[c] = vis ? s[c] * sc : kNegInf;
                mx = fmaxf(mx, s[c]);
            }
            const float m_new = fmaxf(m_ref, mx);
            float alpha = 1.f;
            bool rescale = false;
            if (m_new > m_ref + 8.f) {  // also covers the first visible score (m_ref = -inf)
                alpha = m_ref == kNegInf ? 0.f : ex2(m_ref - m_new);
                rescale = m_ref != kNegInf;
                m_ref = m_new;
            }
            float psum = 0.f;
#pragma unroll
            for (int c = 0; c < BN; ++c) {
                s[c] = m_ref == kNegInf ? 0.f : ex2(s[c] - m_ref);
                psum += s[c];
            }
            l = l * alpha + psum;
            if (i >= 1) {
                ok = __all_sync(0xffffffffu, wait_or_fail(&bars[B_ODONE], (i - 1) & 1, fail, a.status));
                if (!ok) break;
                tc_fence_after();
                // TMEM loads/stores are warp-collective: the warp rescales together,
                // rows whose max did not move scale by one
                if (__any_sync(0xffffffffu, rescale)) {
                    const float f = rescale ? alpha : 1.f;
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
                        float v[32];
                        tmem_ld32(tO + lane_f + 32 * c, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; ++k) v[k] *= f;
                        tmem_st32(tO + lane_f + 32 * c, v);
                    }
                    tmem_wait_st();
                }
            }
#pragma unroll
            for (int q = 0; q < BN / 8; ++q) {
                uint4 u;
                u.x = pack_f16x2(s[8 * q + 0], s[8 * q + 1]);
                u.y = pack_f16x2(s[8 * q + 2], s[8 * q + 3]);
                u.z = pack_f16x2(s[8 * q + 4], s[8 * q + 5]);
                u.w = pack_f16x2(s[8 * q + 6], s[8 * q + 7]);
                *reinterpret_cast<uint4*>(smem + OFF_P + sw128_off(r, 8 * q, REGION)) = u;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            mbar_arrive(&bars[B_PFULL]);
        }
        // ---- epilogue: normalise the O row and store it ----
        if (ok && ntile > 0)
            ok = __all_sync(0xffffffffu, wait_or_fail(&bars[B_ODONE], (ntile - 1) & 1, fail, a.status));
        tc_fence_after();
        float den = l;
        if (a.sink) den += m_ref == kNegInf ? 1.f : ex2(a.sink[h] * kLog2e - m_ref);
        const float inv = den > 0.f ? 1.f / den : 0.f;
        const bool have_o = ok && ntile > 0;  // warp-uniform
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + (((size_t)b * a.T + (valid ? t : 0)) * a.Hq + h) * HD;
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
            float v[32];
            if (have_o) {  // every lane loads (warp-collective); rows past T do not store
                tmem_ld32(tO + lane_f + 32 * c, v);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int k = 0; k < 32; ++k) v[k] = 0.f;
            }
            if (valid) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 u;
                    u.x = pack_bf16x2(v[8 * q + 0] * inv, v[8 * q + 1] * inv);
                    u.y = pack_bf16x2(v[8 * q + 2] * inv, v[8 * q + 3] * inv);
                    u.z = pack_bf16x2(v[8 * q + 4] * inv, v[8 * q + 5] * inv);
                    u.w = pack_bf16x2(v[8 * q + 6] * inv, v[8 * q + 7] * inv);
                    *reinterpret_cast<uint4*>(orow + 32 * c + 8 * q) = u;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

// cos/sin of every (position, pair) the queries and raw keys need.
__global__ void rope_table_kernel(float2* tab, int T, int half, double step) {
    const int64_t n = (int64_t)T * half;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        tab[i] = rope_cs(i / half, (int)(i % half), step);
}

// Finalised raw keys: RoPE at s applied once, fp16 out (the QK^T operand type),
// same [B, T, G, D] layout.
__global__ void finalise_keys_kernel(const __nv_bfloat16* __restrict__ k, __half* __restrict__ out,
                                     const float2* __restrict__ tab, int64_t n_vec, int G, int T, int rho) {
    const int half = rho / 2;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_vec; i += (int64_t)gridDim.x * blockDim.x) {
        const int d0 = (int)(i % (HD / 8)) * 8;
        const int64_t row = i / (HD / 8);            // (b, s, g)
        const int s = (int)((row / G) % T);
        float v[8];
        ld16(k + i * 8, v);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const int d = d0 + e;
            if (d >= HD - rho) rotate_pair(v[e], v[e + 1], tab[(size_t)s * half + ((d - (HD - rho)) >> 1)]);
        }
        st16_f16(out + i * 8, v);
    }
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

size_t prefill_tc_pooled_f16_offset(int B, int T, int G, int rho) {
    const size_t keys = (size_t)B * T * G * HD * 2;
    const size_t tab = (size_t)T * std::max(rho / 2, 1) * sizeof(float2);
    return (keys + 255) / 256 * 256 + (tab + 255) / 256 * 256;
}

// fp16 finalised raw keys, the cos/sin table, and an fp16 copy of the pooled keys
size_t prefill_tc_scratch_bytes(int B, int T, int G, int rho, int m) {
    const size_t pooled = (size_t)B * G * (T / m) * HD * 2;
    return prefill_tc_pooled_f16_offset(B, T, G, rho) + (pooled + 255) / 256 * 256;
}

cudaError_t launch_prefill_tc(const PrefillArgs& p, void* scratch, int32_t* status, cudaStream_t s) {
    if (p.B == 0 || p.T == 0) return cudaSuccess;
    const int G = p.G, T = p.T, B = p.B, Hq = p.Hq;
    __half* keys = static_cast<__half*>(scratch);
    const size_t keys_bytes = ((size_t)B * T * G * HD * 2 + 255) / 256 * 256;
    float2* tab = reinterpret_cast<float2*>(static_cast<char*>(scratch) + keys_bytes);
    const void* pooled_k16 = static_cast<char*>(scratch) + prefill_tc_pooled_f16_offset(B, T, G, p.rho);
    const int half = p.rho / 2;
    if (half > 0) {
        const int64_t n = (int64_t)T * half;
        rope_table_kernel<<<(int)std::min<int64_t>((n + 255) / 256, 148 * 16), 256, 0, s>>>(tab, T, half, p.rope_step);
    }
    {
        const int64_t nv = (int64_t)B * T * G * (HD / 8);
        finalise_keys_kernel<<<(int)std::min<int64_t>((nv + 255) / 256, 148 * 32), 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(p.k), keys, tab, nv, G, T, p.rho);
    }
    TcArgs a;
    memset(&a, 0, sizeof(a));
    const uint64_t e = 2;
    {   // q [B, T, Hq, D]
        const uint64_t dims[4] = {HD, (uint64_t)Hq, (uint64_t)T, (uint64_t)B};
        const uint64_t str[3] = {HD * e, (uint64_t)Hq * HD * e, (uint64_t)T * Hq * HD * e};
        if (!make_map(&a.tq, p.q, dims, str, 1, BM)) return cudaErrorInvalidValue;
    }
    const int NB = T / p.m;
    const uint64_t ps = (uint64_t)std::max(p.pool_stride, 1);
    {   // pooled [B, G, stride, D], valid rows NB
        const uint64_t dims[4] = {HD, (uint64_t)std::max(NB, 1), (uint64_t)G, (uint64_t)B};
        const uint64_t str[3] = {HD * e, ps * HD * e, (uint64_t)G * ps * HD * e};
        if (!make_map(&a.tpv, p.pooled_v, dims, str, BN, 1)) return cudaErrorInvalidValue;
        // fp16 pooled keys in the scratch, [B, G, NB, D]
        const uint64_t nb = (uint64_t)std::max(NB, 1);
        const uint64_t str16[3] = {HD * e, nb * HD * e, (uint64_t)G * nb * HD * e};
        if (!make_map(&a.tpk, pooled_k16, dims, str16, BN, 1, true)) return cudaErrorInvalidValue;
    }
    {   // raw [B, T, G, D]
        const uint64_t dims[4] = {HD, (uint64_t)G, (uint64_t)T, (uint64_t)B};
        const uint64_t str[3] = {HD * e, (uint64_t)G * HD * e, (uint64_t)T * G * HD * e};
        if (!make_map(&a.trk, keys, dims, str, 1, BN, true)) return cudaErrorInvalidValue;
        if (!make_map(&a.trv, p.v, dims, str, 1, BN)) return cudaErrorInvalidValue;
    }
    a.tab = tab;
    a.sink = p.sink;
    a.out = p.out;
    a.status = status;
    a.T = T; a.Hq = Hq; a.G = G; a.m = p.m; a.w = p.w; a.rho = p.rho;
    a.n_qtiles = (T + BM - 1) / BM;
    a.scale = p.scale;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t err = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)SMEM_BYTES);
        if (err != cudaSuccess) return err;
        attr_set = true;
    }
    dim3 grid(Hq, a.n_qtiles, B);
    prefill_tc_kernel<<<grid, 256, SMEM_BYTES, s>>>(a);
    return cudaGetLastError();
}

}  // namespace lbca
