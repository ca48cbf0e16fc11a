// indexer.cu -- lightning-indexer relevance and top-k block selection (the
// CSA form; CSA page, "What is implemented", Eqs 13-17: each indexer head
// scores a compressed indexer key by the ReLU of its dot product with a
// low-rank indexer query, learned per-head weights combine the heads, and the
// k best of the blocks the query may causally see are kept).
//
// For one query per sequence with indexer heads q_h [HI, DI] and head
// weights w_h, the relevance of complete block j is
//     I_j = sum_h w_h ReLU(q_h . k_j),     j < floor(L / m),
// and the k highest-relevance blocks are selected.
//
// B200 mapping.
//   Relevance: the heads' dot products with a tile of 128 compressed keys are
//   one small dense contraction, S^T = K . Q^T (M = 128 key rows, N = HI
//   heads, K = DI), run on tcgen05 with bf16 operands and the f32 result in
//   TMEM; the epilogue thread of TMEM lane r reads its row's HI scores and
//   forms sum_h w_h ReLU(s_h).  A CTA (128 threads) owns one (sequence, tile):
//   the tile and the queries are staged with 16-byte cp.async into
//   128-byte-swizzled shared memory, so each key crosses HBM once.  Several
//   CTAs per SM overlap one tile's copies with another's MMA and epilogue.
//   Top-k: one CTA per sequence holds the relevances in registers as
//   order-preserving 32-bit keys (staged through shared memory so the global
//   reads are coalesced) and finds the k-th largest eight bits at a time (a
//   256-bin histogram per round), then writes the selected block indices in
//   increasing index order (equal relevances: lower index first) followed by
//   -1 padding when fewer than k blocks are visible.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace lbca {
namespace {

constexpr int kRows = 128;       // compressed keys per tile (M of the MMA)
constexpr int kThreads = 128;    // one thread per TMEM lane / key row
constexpr uint64_t kWaitNs = 200ull * 1000 * 1000;

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Relevance of the visible blocks of one 128-row tile.  DI: indexer head dim
// (64 or 128), HI: indexer heads (32, 64 or 128).
template <int DI, int HI>
__global__ void __launch_bounds__(kThreads) indexer_score_kernel(const IndexerArgs a) {
    constexpr int REG_K = kRows * 128;   // one 64-dim column region of the key tile (bytes)
    constexpr int REG_Q = HI * 128;      // one 64-dim column region of the query tile
    constexpr int NREG = DI / 64;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem;                                   // [NREG][128 rows x 128 B]
    uint8_t* sQ = sK + NREG * REG_K;                      // [NREG][HI rows x 128 B]
    float* sw = reinterpret_cast<float*>(sQ + NREG * REG_Q);  // [HI] head weights
    uint64_t* bar = reinterpret_cast<uint64_t*>(sw + HI);
    uint32_t* tmem_sh = reinterpret_cast<uint32_t*>(bar + 1);

    const int tile = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = a.seq_lens[b];
    const int nvis = min(max(L, 0) / a.m, a.max_blocks);
    const int r0 = tile * kRows;
    if (r0 >= nvis) return;  // uniform per CTA: nothing of this tile is visible
    const int nrows = min(kRows, nvis - r0);

    if (warp == 0) tmem_alloc(tmem_sh, HI < 32 ? 32 : HI);
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    // ---- stage the key tile (rows past nrows zero) and the queries, 128B-swizzled ----
    const __nv_bfloat16* kx = static_cast<const __nv_bfloat16*>(a.k_idx) + ((size_t)b * a.max_blocks + r0) * DI;
    const __nv_bfloat16* qx = static_cast<const __nv_bfloat16*>(a.q_idx) + (size_t)b * HI * DI;
    const uint32_t sKa = smem_addr(sK), sQa = smem_addr(sQ);
    for (int c = tid; c < kRows * (DI / 8); c += kThreads) {
        const int r = c / (DI / 8), ch = c % (DI / 8);
        const uint32_t dst = sKa + (uint32_t)(ch >> 3) * REG_K + (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u +
                             ((uint32_t)((ch & 7) ^ (r & 7)) << 4);
        const bool ok = r < nrows;
        cp16(dst, ok ? kx + (size_t)r * DI + ch * 8 : kx, ok ? 16u : 0u);
    }
    for (int c = tid; c < HI * (DI / 8); c += kThreads) {
        const int r = c / (DI / 8), ch = c % (DI / 8);
        const uint32_t dst = sQa + (uint32_t)(ch >> 3) * REG_Q + (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u +
                             ((uint32_t)((ch & 7) ^ (r & 7)) << 4);
        cp16(dst, qx + (size_t)r * DI + ch * 8, 16u);
    }
    for (int h = tid; h < HI; h += kThreads) sw[h] = a.w_idx[(size_t)b * HI + h];
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic-proxy writes -> tensor core reads
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_sh;

    // ---- S^T = K . Q^T: M = 128 key rows, N = HI heads, K = DI, bf16 in, f32 in TMEM ----
    if (tid == 0) {
        constexpr uint32_t idesc = idesc_bf16_f32(kRows, HI, false);
#pragma unroll
        for (int kk = 0; kk < DI / 16; ++kk)
            tc_mma_bf16(tbase, smem_desc_sw128(sKa + (kk >> 2) * REG_K + (kk & 3) * 32, 16, 1024),
                        smem_desc_sw128(sQa + (kk >> 2) * REG_Q + (kk & 3) * 32, 16, 1024), idesc, kk > 0);
        tc_commit(bar);
    }
    bool ok = true;
    if (tid == 0) ok = mbar_wait(bar, 0, kWaitNs);
    ok = __syncthreads_and(ok);
    if (!ok) {
        if (tid == 0) set_status(a.status, LBCA_ERR_TIMEOUT);
    } else {
        // ---- epilogue: TMEM lane = key row; sum_h w_h ReLU(s_h) ----
        tc_fence_after();
        const int row = 32 * warp + lane;
        float acc = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < HI; c0 += 32) {
            float s[32];
            tmem_ld32(tbase + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0, s);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) acc = fmaf(sw[c0 + i], fmaxf(s[i], 0.f), acc);
        }
        if (row < nrows) a.scores[(size_t)b * a.max_blocks + r0 + row] = acc;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, HI < 32 ? 32 : HI);
}

// Order-preserving key of an f32: larger float -> larger unsigned key.
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kKeysPerThread = 32;  // keys held in registers: up to 32768 visible blocks

// Exclusive prefix sum over the CTA (thread order) of one value per thread;
// *total receives the sum over the CTA.
__device__ __forceinline__ unsigned block_exclusive_scan(unsigned v, unsigned* warp_sums, unsigned* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    unsigned before = 0u, all = 0u;
#pragma unroll
    for (int q = 0; q < kSelWarps; ++q) {
        const unsigned w = warp_sums[q];
        before += q < warp ? w : 0u;
        all += w;
    }
    *total = all;
    return before + x - v;
}

// One CTA per sequence.  Thread t holds, as order-preserving keys in
// registers, the relevances of the contiguous run of blocks [t SLOTS, (t + 1)
// SLOTS) (zero keys past the visible blocks), so thread order is block order;
// SLOTS is a compile-time count, so every loop over a thread's keys is exactly
// its keys.  The k-th largest key is found eight bits at a time, most
// significant first (four rounds of a 256-bin histogram of the keys that match
// the digits chosen so far, and one scan of it).  One CTA-wide scan of each
// thread's counts above and equal to the threshold then gives every thread the
// output position of its first taken block: all blocks above the threshold,
// and those equal to it, in block order, until k are taken.
template <int SLOTS>
__global__ void __launch_bounds__(kSelThreads) topk_kernel(const IndexerArgs a) {
    __shared__ unsigned scan_sums[kSelWarps];
    __shared__ uint32_t hist[256];
    __shared__ int sel_round[2];
    const int b = blockIdx.x, tid = threadIdx.x;
    const int L = a.seq_lens[b];
    const int nvis = min(max(L, 0) / a.m, a.max_blocks);
    const int K = a.top_k;
    const float* sc = a.scores + (size_t)b * a.max_blocks;
    int32_t* sel = a.sel + (size_t)b * K;
    float* selv = a.sel_scores ? a.sel_scores + (size_t)b * K : nullptr;

    if (nvis <= K) {  // every visible block is selected
        for (int i = tid; i < K; i += kSelThreads) {
            sel[i] = i < nvis ? i : -1;
            if (selv) selv[i] = i < nvis ? sc[i] : kNegInf;
        }
        return;
    }
    if (nvis > kSelThreads * SLOTS) {  // beyond the register capacity (the host sizes forbid it)
        if (tid == 0) set_status(a.status, LBCA_ERR_CAPACITY);
        for (int i = tid; i < K; i += kSelThreads) sel[i] = -1;
        return;
    }
    // the relevances pass through shared memory: read from global in block order
    // (coalesced), then each thread takes its contiguous run (one padding word
    // per run keeps the runs on different banks)
    extern __shared__ float stage[];  // kSelThreads runs of SLOTS + 1 words
    for (int i = tid; i < nvis; i += kSelThreads) stage[i + i / SLOTS] = sc[i];
    __syncthreads();
    const int i0 = tid * SLOTS;
    uint32_t key[SLOTS];
#pragma unroll
    for (int s = 0; s < SLOTS; ++s)
        key[s] = i0 + s < nvis ? order_key(stage[tid * (SLOTS + 1) + s]) : 0u;  // 0: below every real key
    // ---- the k-th largest key, eight bits at a time ----
    // Round r histograms digit r (most significant first) of the keys that match
    // the digits chosen so far; the lanes of a warp holding lane 0's digit add
    // once (a ballot), so keys that share their top bits (most relevances do) do
    // not serialise the shared-memory adds.  The digit whose bin holds the k-th largest of those
    // keys is kept, and k is reduced by the keys in the bins above it.
    uint32_t thr = 0u, tmask = 0u;
    int need = K;
    const int lane = tid & 31;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0u;
        if (tid == 0) sel_round[0] = sel_round[1] = 0;
        __syncthreads();
#pragma unroll
        for (int s = 0; s < SLOTS; ++s) {
            const bool in = i0 + s < nvis && (key[s] & tmask) == thr;
            const uint32_t dg = in ? (key[s] >> shift) & 255u : 256u;
            // the lanes that share lane 0's digit add once; the others one by one
            const uint32_t d0 = __shfl_sync(0xffffffffu, dg, 0);
            const uint32_t same = __ballot_sync(0xffffffffu, dg == d0);
            if (lane == 0 && d0 != 256u) atomicAdd(&hist[d0], (uint32_t)__popc(same));
            if (dg != d0 && in) atomicAdd(&hist[dg], 1u);
        }
        __syncthreads();
        if (tid < 32) {  // warp 0: lane l holds bins [8l, 8l + 8); scan from the top
            uint32_t h[8], tot = 0u;
#pragma unroll
            for (int q = 0; q < 8; ++q) { h[q] = hist[8 * tid + q]; tot += h[q]; }
            // keys in the bins of the lanes above this one: an inclusive suffix sum
            // (log-step) minus this lane's own bins
            uint32_t suf = tot;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t y = __shfl_down_sync(0xffffffffu, suf, off);
                if (tid + off < 32) suf += y;
            }
            uint32_t above = suf - tot;
            for (int q = 7; q >= 0; --q) {
                if (above < (uint32_t)need && (uint32_t)need <= above + h[q]) {
                    sel_round[0] = 8 * tid + q;
                    sel_round[1] = (int)above;
                }
                above += h[q];
            }
        }
        __syncthreads();
        thr |= (uint32_t)sel_round[0] << shift;
        tmask |= 255u << shift;
        need -= sel_round[1];
        __syncthreads();  // hist and sel_round are rewritten by the next round
    }
    // ---- counts above and at the threshold, one scan of both (16-bit halves) ----
    int gt = 0, eq = 0;
#pragma unroll
    for (int s = 0; s < SLOTS; ++s) {
        gt += key[s] > thr;
        eq += key[s] == thr && i0 + s < nvis;
    }
    unsigned all = 0u;  // each half sums at most 32768
    const unsigned packed = block_exclusive_scan((unsigned)gt | ((unsigned)eq << 16), scan_sums, &all);
    const int gt_before = (int)(packed & 0xffffu), eq_before = (int)(packed >> 16);
    const int ties_needed = K - (int)(all & 0xffffu);
    // ---- this thread's blocks, in order ----
    int pos = gt_before + min(eq_before, ties_needed);
    int ties_seen = eq_before;
#pragma unroll
    for (int s = 0; s < SLOTS; ++s) {
        const int i = i0 + s;
        const bool tie = i < nvis && key[s] == thr;
        const bool take = key[s] > thr || (tie && ties_seen < ties_needed);
        ties_seen += tie ? 1 : 0;
        if (take && pos < K) {
            sel[pos] = i;
            if (selv) selv[pos] = __uint_as_float(key[s] & 0x80000000u ? key[s] & 0x7fffffffu : ~key[s]);
        }
        pos += take ? 1 : 0;
    }
    if (tid == kSelThreads - 1 && pos != K) set_status(a.status, LBCA_ERR_ARG);  // cannot happen: the select is exact
}

template <int SLOTS>
cudaError_t launch_topk(const IndexerArgs& a, cudaStream_t s) {
    const size_t smem = (size_t)kSelThreads * (SLOTS + 1) * sizeof(float);
    static bool attr[64] = {};  // per device
    const int dev_ = current_device();
    if (dev_ < 0 || !attr[dev_]) {
        cudaError_t e = cudaFuncSetAttribute(topk_kernel<SLOTS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev_ >= 0) attr[dev_] = true;
    }
    topk_kernel<SLOTS><<<a.B, kSelThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <int DI, int HI>
size_t score_smem() {
    return (size_t)DI / 64 * (kRows + HI) * 128 + HI * 4 + 64 + 1024;
}

template <int DI, int HI>
cudaError_t launch_score(const IndexerArgs& a, cudaStream_t s) {
    const size_t smem = score_smem<DI, HI>();
    static bool attr[64] = {};  // per device
    const int dev_ = current_device();
    if (dev_ < 0 || !attr[dev_]) {
        cudaError_t e = cudaFuncSetAttribute(indexer_score_kernel<DI, HI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        if (dev_ >= 0) attr[dev_] = true;
    }
    dim3 grid((a.max_blocks + kRows - 1) / kRows, a.B);
    indexer_score_kernel<DI, HI><<<grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool indexer_shape_ok(int HI, int DI) {
    return (DI == 64 || DI == 128) && (HI == 32 || HI == 64 || HI == 128);
}

cudaError_t launch_indexer_topk(const IndexerArgs& a, cudaStream_t s) {
    if (a.B == 0) return cudaSuccess;
    if (a.B > 65535) return cudaErrorInvalidValue;
    cudaError_t e = cudaSuccess;
    if (a.max_blocks > 0) {
        if (a.DI == 64) {
            e = a.HI == 32 ? launch_score<64, 32>(a, s) : a.HI == 64 ? launch_score<64, 64>(a, s)
                                                                      : launch_score<64, 128>(a, s);
        } else {
            e = a.HI == 32 ? launch_score<128, 32>(a, s) : a.HI == 64 ? launch_score<128, 64>(a, s)
                                                                       : launch_score<128, 128>(a, s);
        }
        if (e != cudaSuccess) return e;
    }
    // the fewest register slots that hold every visible block of any sequence
    const int need = (a.max_blocks + kSelThreads - 1) / kSelThreads;
    if (need <= 1) return launch_topk<1>(a, s);
    if (need <= 2) return launch_topk<2>(a, s);
    if (need <= 4) return launch_topk<4>(a, s);
    if (need <= 8) return launch_topk<8>(a, s);
    if (need <= 16) return launch_topk<16>(a, s);
    return launch_topk<kKeysPerThread>(a, s);
}

}  // namespace lbca
