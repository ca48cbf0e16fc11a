// api.cu -- the C ABI: argument validation, device check, launches.
//
// Every entry point validates its arguments on the host before any CUDA call
// (so bad arguments are reported even without a GPU), checks that the current
// device is sm_100, and enqueues its kernels on the caller's stream.  No entry
// point allocates device memory or synchronises.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "lbca.h"

using namespace lbca;

namespace {

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool al16n(const void* p) { return p == nullptr || al16(p); }

int vec_of(int dtype) { return dtype == LBCA_BF16 ? 8 : 4; }
int esize_of(int dtype) { return dtype == LBCA_BF16 ? 2 : 4; }

lbca_status check_cfg(const lbca_config* c) {
    if (!c) return LBCA_ERR_ARG;
    if (c->n_q_heads < 1 || c->n_kv_heads < 1 || c->n_q_heads % c->n_kv_heads) return LBCA_ERR_ARG;
    if (c->head_dim < 16 || c->head_dim > 512 || c->head_dim % 16) return LBCA_ERR_ARG;
    if ((c->shared_kv != 0 && c->shared_kv != 1) || (c->rmsnorm != 0 && c->rmsnorm != 1)) return LBCA_ERR_ARG;
    if (c->block_m < 1 || c->n_win < 0) return LBCA_ERR_ARG;
    if (c->rope_dims < 0 || c->rope_dims > c->head_dim || (c->rope_dims & 1)) return LBCA_ERR_ARG;
    if (c->rope_dims > 0 && !(c->rope_theta > 0.0)) return LBCA_ERR_ARG;
    if (c->rmsnorm && !(c->rms_eps >= 0.f)) return LBCA_ERR_ARG;
    if (!(c->softmax_scale == c->softmax_scale)) return LBCA_ERR_ARG;  // NaN
    if (c->dtype != LBCA_F32 && c->dtype != LBCA_BF16) return LBCA_ERR_ARG;
    if (c->reserved != 0) return LBCA_ERR_ARG;
    // pooling kernels keep one 16-byte vector of the G*D row per thread (<= 1024 threads)
    const long long nv = (long long)c->n_kv_heads * c->head_dim / vec_of(c->dtype);
    if (nv * (c->shared_kv ? 1 : 2) > 1024) return LBCA_ERR_UNSUPPORTED;
    return LBCA_OK;
}

float scale_of(const lbca_config* c) {
    return c->softmax_scale > 0.f ? c->softmax_scale : 1.0f / std::sqrt((float)c->head_dim);
}

// theta^(-2/rho): pair k of the rotated dims turns by step^k radians per position
double rope_step_of(const lbca_config* c) {
    return c->rope_dims > 0 ? std::pow(c->rope_theta, -2.0 / (double)c->rope_dims) : 1.0;
}

int ring_min(const lbca_config* c) {
    const long long m = c->block_m;
    long long r = m * ((c->n_win + m - 1 + m - 1) / m);
    if (r < 1) r = 1;
    return r > INT32_MAX ? -1 : (int)r;
}

lbca_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LBCA_ERR_CUDA;
    static int known[64];  // 0 unknown, 1 sm_100, 2 other
    if (dev >= 0 && dev < 64 && known[dev]) return known[dev] == 1 ? LBCA_OK : LBCA_ERR_UNSUPPORTED;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return LBCA_ERR_CUDA;
    const bool ok = major == 10 && minor == 0;
    if (dev >= 0 && dev < 64) known[dev] = ok ? 1 : 2;
    return ok ? LBCA_OK : LBCA_ERR_UNSUPPORTED;
}

lbca_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LBCA_OK : LBCA_ERR_CUDA; }

lbca_status check_cache(const lbca_config* c, const lbca_cache* k) {
    if (!k) return LBCA_ERR_ARG;
    if (k->batch < 0 || k->max_blocks < 0 || (k->flags & ~LBCA_CACHE_OVERLAP_PREV) != 0) return LBCA_ERR_ARG;
    const int rmin = ring_min(c);
    if (rmin < 0 || k->ring_slots < rmin) return LBCA_ERR_CAPACITY;
    const bool pooled = k->max_blocks > 0;  // a cache with no block capacity needs no pooled arrays
    if ((pooled && !k->pooled_k) || !k->ring_k || !k->pool_state || !k->seq_lens) return LBCA_ERR_ARG;
    if (c->shared_kv) {
        if (k->pooled_v || k->ring_v) return LBCA_ERR_ARG;
    } else if ((pooled && !k->pooled_v) || !k->ring_v) {
        return LBCA_ERR_ARG;
    }
    if (!al16(k->pooled_k) || !al16n(k->pooled_v) || !al16(k->ring_k) || !al16n(k->ring_v) ||
        !al16(k->pool_state))
        return LBCA_ERR_ALIGN;
    return LBCA_OK;
}

// K-side / V-side pointer set: shared form needs exactly the K side.
// `need_tokens` is false for a zero-token prefill, whose k, v, zk, zv may be NULL.
lbca_status check_kv(const lbca_config* c, const void* k, const void* v, const void* zk, const void* zv,
                     const void* bk, const void* bv, bool need_tokens = true) {
    if ((need_tokens && (!k || !zk)) || !bk) return LBCA_ERR_ARG;
    if (c->shared_kv) {
        if (v || zv || bv) return LBCA_ERR_ARG;
    } else if ((need_tokens && (!v || !zv)) || !bv) {
        return LBCA_ERR_ARG;
    }
    if (!al16(k) || !al16(zk) || !al16(bk) || !al16n(v) || !al16n(zv) || !al16n(bv)) return LBCA_ERR_ALIGN;
    return LBCA_OK;
}

#define LBCA_TRY(expr)                    \
    do {                                  \
        lbca_status _s = (expr);          \
        if (_s != LBCA_OK) return _s;     \
    } while (0)

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Decode arguments common to every decode launch (no workspace, no split plan).
DecodeArgs decode_args(const lbca_config* cfg, const void* q, const lbca_cache* cache, const float* sink,
                       const void* gamma_q, const void* gamma_kv, void* out, int32_t* d_status) {
    DecodeArgs a{};
    a.dtype = cfg->dtype;
    a.q = q;
    a.pooled_k = cache->pooled_k; a.pooled_v = cache->pooled_v;
    a.ring_k = cache->ring_k; a.ring_v = cache->ring_v;
    a.seq_lens = cache->seq_lens; a.sink = sink; a.gamma_q = gamma_q; a.gamma_kv = gamma_kv; a.out = out;
    a.status = d_status;
    a.B = cache->batch; a.Hq = cfg->n_q_heads; a.G = cfg->n_kv_heads; a.D = cfg->head_dim;
    a.m = cfg->block_m; a.w = cfg->n_win; a.rho = cfg->rope_dims; a.rmsnorm = cfg->rmsnorm;
    a.shared = cfg->shared_kv; a.max_blocks = cache->max_blocks; a.R = cache->ring_slots;
    a.eps = cfg->rms_eps; a.scale = scale_of(cfg); a.rope_step = rope_step_of(cfg);
    return a;
}

// The serving step of the shared-entry form on the tensor-core kernel with the
// append fused in: bf16, one kv head and a raw window (so an entry finished
// by this step's token is not yet visible to its query).  Shape tests only.
bool step_mqa_fused(const lbca_config* c, int batch, int max_ctx) {
    return c->n_kv_heads == 1 && c->n_win >= 1 &&
           mqa_tc_shape_ok(c->dtype, batch, c->n_q_heads, c->n_kv_heads, c->head_dim, c->block_m, c->n_win,
                           c->shared_kv, max_ctx);
}

// The decode launch: the tensor-core kernel for the shared-entry form where it
// applies (it needs no workspace), else the CUDA-core split-KV kernel.
lbca_status run_decode(const lbca_config* cfg, DecodeArgs& a, int32_t max_ctx, cudaStream_t s) {
    const MqaTcPlan tc = plan_decode_mqa_tc(cfg->dtype, a.B, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim,
                                            cfg->block_m, cfg->n_win, cfg->shared_kv, max_ctx);
    a.tc_cs = tc.cs;
    if (tc.cs > 0) {
        a.chunk = tc.rows;
        return cuda_status(launch_decode_mqa_tc(a, s));
    }
    return cuda_status(launch_decode(a, s));
}

}  // namespace

extern "C" {

int32_t lbca_ring_slots(const lbca_config* cfg) {
    if (check_cfg(cfg) != LBCA_OK) return -1;
    return ring_min(cfg);
}

size_t lbca_pool_state_elems(const lbca_config* cfg, int32_t batch) {
    if (check_cfg(cfg) != LBCA_OK || batch < 0) return 0;
    return (size_t)batch * (cfg->shared_kv ? 1 : 2) * 3 * cfg->n_kv_heads * cfg->head_dim;
}

size_t lbca_decode_workspace_bytes(const lbca_config* cfg, int32_t batch, int32_t max_ctx) {
    if (check_cfg(cfg) != LBCA_OK || batch < 0 || max_ctx < 1) return 0;
    DecodePlan p = plan_decode(cfg->dtype, batch, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim,
                               cfg->block_m, cfg->n_win, cfg->shared_kv, max_ctx);
    if (!p.ok) return 0;
    return decode_workspace_bytes(p);
}

size_t lbca_prefill_workspace_bytes(const lbca_config* cfg, int32_t batch, int32_t T, int32_t has_cache) {
    if (check_cfg(cfg) != LBCA_OK || batch < 0 || T < 0) return (size_t)-1;
    size_t bytes = 0;
    if (!has_cache) {
        const size_t one = (size_t)batch * cfg->n_kv_heads * (T / cfg->block_m) * cfg->head_dim *
                           esize_of(cfg->dtype);
        bytes = align256(one) * (cfg->shared_kv ? 1 : 2);
    }
    if (prefill_tc_supported(cfg->dtype, cfg->head_dim, cfg->rmsnorm, cfg->shared_kv))
        bytes += align256(prefill_tc_scratch_bytes(batch, T, cfg->n_kv_heads, cfg->rope_dims, cfg->block_m));
    return bytes;
}

// Fields common to every pooling call of blocks [pos0/m, pos0/m + T/m).
static void pool_common(const lbca_config* cfg, int32_t batch, int32_t T, int32_t pos0, int32_t out_blocks,
                        PoolArgs& a) {
    a.dtype = cfg->dtype;
    a.out_blocks = out_blocks; a.blk_off = pos0 / cfg->block_m;
    a.B = batch; a.T = T; a.G = cfg->n_kv_heads; a.D = cfg->head_dim; a.m = cfg->block_m;
    a.pos0 = pos0;
    a.rmsnorm = cfg->rmsnorm; a.rho = cfg->rope_dims;
    a.rope_step = rope_step_of(cfg); a.eps = cfg->rms_eps;
    a.state = nullptr; a.S = 1;
}

// One series pooled into `out` (the I/O dtype) or `out_f32` (f32 entries).
static lbca_status pool_single(const lbca_config* cfg, int32_t series, const void* x, const void* z,
                               const void* b_pos, const void* gamma, int32_t batch, int32_t T, int32_t pos0,
                               void* out, float* out_f32, int32_t out_blocks, lbca_stream_t stream) {
    LBCA_TRY(check_cfg(cfg));
    if (!out && !out_f32) return LBCA_ERR_ARG;
    if (series != LBCA_KEY && series != LBCA_VALUE) return LBCA_ERR_ARG;
    if (cfg->shared_kv && series != LBCA_KEY) return LBCA_ERR_ARG;
    if (!x || !z || !b_pos) return LBCA_ERR_ARG;
    if (batch < 0 || T < 0 || pos0 < 0 || pos0 % cfg->block_m || out_blocks < 0) return LBCA_ERR_ARG;
    if ((long long)pos0 / cfg->block_m + T / cfg->block_m > out_blocks) return LBCA_ERR_ARG;
    if (!al16(x) || !al16(z) || !al16(b_pos) || !al16n(out) || !al16n(out_f32) || !al16n(gamma))
        return LBCA_ERR_ALIGN;
    LBCA_TRY(check_device());
    PoolArgs a{};
    pool_common(cfg, batch, T, pos0, out_blocks, a);
    a.nser = 1;
    a.ser[0].x = x; a.ser[0].z = z; a.ser[0].bpos = b_pos; a.ser[0].gamma = gamma;
    // f32 I/O: the entries are f32 already
    a.ser[0].out = out ? out : (cfg->dtype == LBCA_F32 ? out_f32 : nullptr);
    a.ser[0].out_f32 = cfg->dtype == LBCA_F32 ? nullptr : out_f32;
    a.ser[0].key = series == LBCA_KEY; a.ser[0].state_series = 0;
    return cuda_status(launch_pool(a, reinterpret_cast<cudaStream_t>(stream)));
}

lbca_status lbca_pool(const lbca_config* cfg, int32_t series, const void* x, const void* z,
                      const void* b_pos, const void* gamma, int32_t batch, int32_t T, int32_t pos0,
                      void* out, int32_t out_blocks, lbca_stream_t stream) {
    if (!out) return LBCA_ERR_ARG;
    return pool_single(cfg, series, x, z, b_pos, gamma, batch, T, pos0, out, nullptr, out_blocks, stream);
}

lbca_status lbca_pool_f32(const lbca_config* cfg, int32_t series, const void* x, const void* z,
                          const void* b_pos, const void* gamma, int32_t batch, int32_t T, int32_t pos0,
                          float* out, int32_t out_blocks, lbca_stream_t stream) {
    if (!out) return LBCA_ERR_ARG;
    return pool_single(cfg, series, x, z, b_pos, gamma, batch, T, pos0, nullptr, out, out_blocks, stream);
}

lbca_status lbca_pool_kv(const lbca_config* cfg, const void* k, const void* v, const void* zk, const void* zv,
                         const void* b_pos_k, const void* b_pos_v, const void* gamma_kv, int32_t batch, int32_t T,
                         int32_t pos0, void* pooled_k, void* pooled_v, int32_t out_blocks, lbca_stream_t stream) {
    LBCA_TRY(check_cfg(cfg));
    if (cfg->shared_kv) return LBCA_ERR_ARG;
    if (!k || !v || !zk || !zv || !b_pos_k || !b_pos_v || !pooled_k || !pooled_v) return LBCA_ERR_ARG;
    if (batch < 0 || T < 0 || pos0 < 0 || pos0 % cfg->block_m || out_blocks < 0) return LBCA_ERR_ARG;
    if ((long long)pos0 / cfg->block_m + T / cfg->block_m > out_blocks) return LBCA_ERR_ARG;
    if (!al16(k) || !al16(v) || !al16(zk) || !al16(zv) || !al16(b_pos_k) || !al16(b_pos_v) || !al16(pooled_k) ||
        !al16(pooled_v) || !al16n(gamma_kv))
        return LBCA_ERR_ALIGN;
    LBCA_TRY(check_device());
    PoolArgs a{};
    pool_common(cfg, batch, T, pos0, out_blocks, a);
    a.nser = 2;
    for (int series = 0; series < 2; ++series) {
        PoolSeries& sr = a.ser[series];
        sr.x = series ? v : k; sr.z = series ? zv : zk; sr.bpos = series ? b_pos_v : b_pos_k;
        sr.gamma = series ? nullptr : gamma_kv;
        sr.out = series ? pooled_v : pooled_k;
        sr.key = series == 0; sr.state_series = series;
    }
    return cuda_status(launch_pool(a, reinterpret_cast<cudaStream_t>(stream)));
}

lbca_status lbca_pool_dual(const lbca_config* cfg, int32_t series, const void* xa, const void* za, const void* xb,
                           const void* zb, const void* b_pos_a, const void* b_pos_b, const void* gamma, int32_t batch,
                           int32_t T, void* out, int32_t out_blocks, lbca_stream_t stream) {
    LBCA_TRY(check_cfg(cfg));
    if (series != LBCA_KEY && series != LBCA_VALUE) return LBCA_ERR_ARG;
    if (!xa || !za || !xb || !zb || !b_pos_a || !b_pos_b || !out) return LBCA_ERR_ARG;
    if (batch < 0 || T < 0 || out_blocks < 0 || T / cfg->block_m > out_blocks) return LBCA_ERR_ARG;
    if (!al16(xa) || !al16(za) || !al16(xb) || !al16(zb) || !al16(b_pos_a) || !al16(b_pos_b) || !al16(out) ||
        !al16n(gamma))
        return LBCA_ERR_ALIGN;
    LBCA_TRY(check_device());
    PoolArgs a{};
    a.dtype = cfg->dtype;
    a.nser = 1;
    a.dual = 1;
    PoolSeries& sr = a.ser[0];
    sr.x = xa; sr.z = za; sr.bpos = b_pos_a; sr.xb = xb; sr.zb = zb; sr.bposb = b_pos_b;
    sr.gamma = gamma; sr.out = out; sr.key = series == LBCA_KEY;
    a.out_blocks = out_blocks; a.blk_off = 0;
    a.B = batch; a.T = T; a.G = cfg->n_kv_heads; a.D = cfg->head_dim; a.m = cfg->block_m; a.pos0 = 0;
    a.rmsnorm = cfg->rmsnorm; a.rho = cfg->rope_dims; a.rope_step = rope_step_of(cfg); a.eps = cfg->rms_eps;
    a.S = 1;
    return cuda_status(launch_pool(a, reinterpret_cast<cudaStream_t>(stream)));
}

lbca_status lbca_append(const lbca_config* cfg, const void* k, const void* v, const void* zk,
                        const void* zv, const void* b_pos_k, const void* b_pos_v, const void* gamma_kv,
                        const lbca_cache* cache, int32_t* d_status, lbca_stream_t stream) {
    LBCA_TRY(check_cfg(cfg));
    LBCA_TRY(check_kv(cfg, k, v, zk, zv, b_pos_k, b_pos_v));
    LBCA_TRY(check_cache(cfg, cache));
    if (!al16n(gamma_kv)) return LBCA_ERR_ALIGN;
    LBCA_TRY(check_device());
    AppendArgs a{};
    a.dtype = cfg->dtype;
    a.k = k; a.v = v; a.zk = zk; a.zv = zv; a.bpk = b_pos_k; a.bpv = b_pos_v; a.gamma = gamma_kv;
    a.pooled_k = cache->pooled_k; a.pooled_v = cache->pooled_v;
    a.ring_k = cache->ring_k; a.ring_v = cache->ring_v;
    a.state = cache->pool_state; a.seq_lens = cache->seq_lens; a.status = d_status;
    a.B = cache->batch; a.G = cfg->n_kv_heads; a.D = cfg->head_dim; a.m = cfg->block_m;
    a.R = cache->ring_slots; a.max_blocks = cache->max_blocks; a.S = cfg->shared_kv ? 1 : 2;
    a.rmsnorm = cfg->rmsnorm; a.rho = cfg->rope_dims; a.rope_step = rope_step_of(cfg); a.eps = cfg->rms_eps;
    return cuda_status(launch_append(a, reinterpret_cast<cudaStream_t>(stream)));
}

lbca_status lbca_decode(const lbca_config* cfg, const void* q, const lbca_cache* cache, const float* sink,
                        const void* gamma_q, const void* gamma_kv, int32_t max_ctx, void* out, void* workspace,
                        size_t workspace_bytes, int32_t* d_status, lbca_stream_t stream) {
    LBCA_TRY(check_cfg(cfg));
    LBCA_TRY(check_cache(cfg, cache));
    if (!q || !out || !workspace) return LBCA_ERR_ARG;
    if (!al16(q) || !al16(out) || !al16(workspace) || !al16n(gamma_q) || !al16n(gamma_kv) || !al16n(sink))
        return LBCA_ERR_ALIGN;
    if (max_ctx <= 0) {
        const long long cap = (long long)cache->max_blocks * cfg->block_m + cache->ring_slots;
        max_ctx = cap > INT32_MAX ? INT32_MAX : (int32_t)(cap < 1 ? 1 : cap);
    }
    DecodePlan p = plan_decode(cfg->dtype, cache->batch, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim,
                               cfg->block_m, cfg->n_win, cfg->shared_kv, max_ctx);
    if (!p.ok) return LBCA_ERR_UNSUPPORTED;
    if (workspace_bytes < decode_workspace_bytes(p)) return LBCA_ERR_CAPACITY;
    LBCA_TRY(check_device());
    char* ws = static_cast<char*>(workspace);
    DecodeArgs a = decode_args(cfg, q, cache, sink, gamma_q, gamma_kv, out, d_status);
    a.part_o = reinterpret_cast<float*>(ws);
    a.part_ml = reinterpret_cast<float*>(ws + align256(p.part_o_elems * 4));
    a.counters = reinterpret_cast<uint32_t*>(ws + align256(p.part_o_elems * 4) + align256(p.part_ml_elems * 4));
    a.n_split = p.n_split; a.chunk = p.chunk; a.heads_per_cta = p.heads_per_cta;
    return run_decode(cfg, a, max_ctx, reinterpret_cast<cudaStream_t>(stream));
}

size_t lbca_decode_step_workspace_bytes(const lbca_config* cfg, int32_t batch, int32_t max_ctx) {
    if (check_cfg(cfg) != LBCA_OK || batch < 0 || max_ctx < 1) return 0;
    if (step_mqa_fused(cfg, batch, max_ctx)) return 256;  // the fused tensor-core step uses none
    StepPlan sp = plan_step(cfg->dtype, batch, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim, cfg->block_m,
                            cfg->n_win, cfg->shared_kv, max_ctx);
    if (sp.ok) return step_workspace_bytes(sp);
    return lbca_decode_workspace_bytes(cfg, batch, max_ctx);  // append + decode fallback
}

int32_t lbca_decode_step_launches(const lbca_config* cfg, int32_t batch, int32_t max_ctx) {
    if (check_cfg(cfg) != LBCA_OK || batch < 0 || max_ctx < 1) return -1;
    const StepPlan sp = plan_step(cfg->dtype, batch, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim, cfg->block_m,
                                  cfg->n_win, cfg->shared_kv, max_ctx);
    return (step_mqa_fused(cfg, batch, max_ctx) || sp.ok) ? 1 : 2;
}

int32_t lbca_decode_step_form(const lbca_config* cfg, int32_t batch, int32_t max_ctx) {
    if (check_cfg(cfg) != LBCA_OK || batch < 0 || max_ctx < 1) return -1;
    const StepPlan sp = plan_step(cfg->dtype, batch, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim, cfg->block_m,
                                  cfg->n_win, cfg->shared_kv, max_ctx);
    if (step_mqa_fused(cfg, batch, max_ctx)) return LBCA_STEP_SHARED_TC;
    if (!sp.ok) return LBCA_STEP_TWO_CALLS;
    return sp.flat ? LBCA_STEP_PERSISTENT : LBCA_STEP_CLUSTER;
}

lbca_status lbca_decode_step(const lbca_config* cfg, const void* k, const void* v, const void* zk, const void* zv,
                             const void* b_pos_k, const void* b_pos_v, const void* gamma_kv, const void* q,
                             const lbca_cache* cache, const float* sink, const void* gamma_q, int32_t max_ctx,
                             void* out, void* workspace, size_t workspace_bytes, int32_t* d_status,
                             lbca_stream_t stream) {
    LBCA_TRY(check_cfg(cfg));
    LBCA_TRY(check_kv(cfg, k, v, zk, zv, b_pos_k, b_pos_v));
    LBCA_TRY(check_cache(cfg, cache));
    if (!q || !out || !workspace) return LBCA_ERR_ARG;
    if (!al16(q) || !al16(out) || !al16(workspace) || !al16n(gamma_q) || !al16n(gamma_kv) || !al16n(sink))
        return LBCA_ERR_ALIGN;
    if (max_ctx <= 0) {
        const long long cap = (long long)cache->max_blocks * cfg->block_m + cache->ring_slots;
        max_ctx = cap > INT32_MAX ? INT32_MAX : (int32_t)(cap < 1 ? 1 : cap);
    }
    if (step_mqa_fused(cfg, cache->batch, max_ctx)) {  // shared-entry tensor-core decode, append fused
        LBCA_TRY(check_device());
        const MqaTcPlan tp = plan_decode_mqa_tc(cfg->dtype, cache->batch, cfg->n_q_heads, cfg->n_kv_heads,
                                                cfg->head_dim, cfg->block_m, cfg->n_win, cfg->shared_kv, max_ctx);
        if (tp.cs == 0) return LBCA_ERR_UNSUPPORTED;  // no cluster of the kernel fits this device
        DecodeArgs a = decode_args(cfg, q, cache, sink, gamma_q, gamma_kv, out, d_status);
        a.app_k = k; a.app_z = zk; a.app_bp = b_pos_k;
        a.ring_w = cache->ring_k; a.pooled_w = cache->pooled_k; a.state = cache->pool_state;
        a.lens_w = cache->seq_lens;
        a.tc_cs = tp.cs; a.chunk = tp.rows;
        a.pdl = (cache->flags & LBCA_CACHE_OVERLAP_PREV) != 0;
        return cuda_status(launch_decode_mqa_tc(a, reinterpret_cast<cudaStream_t>(stream)));
    }
    StepPlan sp = plan_step(cfg->dtype, cache->batch, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim,
                            cfg->block_m, cfg->n_win, cfg->shared_kv, max_ctx);
    if (!sp.ok) {  // shapes no fused kernel takes: the two-launch path
        LBCA_TRY(lbca_append(cfg, k, v, zk, zv, b_pos_k, b_pos_v, gamma_kv, cache, d_status, stream));
        return lbca_decode(cfg, q, cache, sink, gamma_q, gamma_kv, max_ctx, out, workspace, workspace_bytes,
                           d_status, stream);
    }
    if (workspace_bytes < step_workspace_bytes(sp)) return LBCA_ERR_CAPACITY;
    LBCA_TRY(check_device());
    StepArgs a{};
    a.dtype = cfg->dtype;
    a.k = k; a.v = v; a.zk = zk; a.zv = zv; a.bpk = b_pos_k; a.bpv = b_pos_v; a.gamma_kv = gamma_kv;
    a.q = q; a.sink = sink; a.gamma_q = gamma_q; a.out = out;
    a.pooled_k = cache->pooled_k; a.pooled_v = cache->pooled_v; a.ring_k = cache->ring_k; a.ring_v = cache->ring_v;
    a.state = cache->pool_state; a.seq_lens = cache->seq_lens;
    a.arrive = static_cast<uint32_t*>(workspace); a.status = d_status;
    a.B = cache->batch; a.Hq = cfg->n_q_heads; a.G = cfg->n_kv_heads; a.D = cfg->head_dim; a.m = cfg->block_m;
    a.w = cfg->n_win; a.rho = cfg->rope_dims; a.rmsnorm = cfg->rmsnorm; a.shared = cfg->shared_kv;
    a.max_blocks = cache->max_blocks; a.R = cache->ring_slots; a.S = cfg->shared_kv ? 1 : 2;
    a.CS = sp.CS; a.SE = sp.SE; a.heads_per_cta = sp.heads_per_cta;
    a.pdl = (cache->flags & LBCA_CACHE_OVERLAP_PREV) != 0;
    a.eps = cfg->rms_eps; a.scale = scale_of(cfg); a.rope_step = rope_step_of(cfg);
    if (sp.flat) {
        for (int kk = 0; kk < cfg->rope_dims / 2 && kk < 128; ++kk) a.rope_f[kk] = rope_turns(kk, a.rope_step);
        // workspace: [arrival counter][segment counters][partial max, sum][partial outputs]
        char* ws = static_cast<char*>(workspace);
        const size_t o1 = align256(4), o2 = o1 + align256(sp.seg_elems * 4), o3 = o2 + align256(sp.part_ml_elems * 4);
        a.seg_count = reinterpret_cast<uint32_t*>(ws + o1);
        a.part_ml = reinterpret_cast<float*>(ws + o2);
        a.part_o = reinterpret_cast<float*>(ws + o3);
        a.C = sp.C;
        a.maxc = sp.maxc;
        LBCA_TRY(cuda_status(flat_grid(&a.grid, a.dtype, a.D, a.heads_per_cta, sp.smem_bytes)));
    }
    return cuda_status(launch_decode_step(a, reinterpret_cast<cudaStream_t>(stream)));
}

lbca_status lbca_prefill(const lbca_config* cfg, const void* q, const void* k, const void* v, const void* zk,
                         const void* zv, const void* b_pos_k, const void* b_pos_v, const float* sink,
                         const void* gamma_q, const void* gamma_kv, int32_t batch, int32_t T, void* out,
                         const lbca_cache* cache_out, void* workspace, size_t workspace_bytes,
                         int32_t* d_status, lbca_stream_t stream) {
    LBCA_TRY(check_cfg(cfg));
    if (batch < 0 || T < 0) return LBCA_ERR_ARG;
    LBCA_TRY(check_kv(cfg, k, v, zk, zv, b_pos_k, b_pos_v, T > 0 && batch > 0));
    if (!out && !cache_out) return LBCA_ERR_ARG;
    if (out && !q) return LBCA_ERR_ARG;
    if (!al16n(q) || !al16n(out) || !al16n(gamma_q) || !al16n(gamma_kv) || !al16n(sink) ||
        !al16n(workspace))
        return LBCA_ERR_ALIGN;
    const int m = cfg->block_m, NB = T / m;
    if (cache_out) {
        LBCA_TRY(check_cache(cfg, cache_out));
        if (cache_out->batch != batch) return LBCA_ERR_ARG;
        if (cache_out->max_blocks < NB) return LBCA_ERR_CAPACITY;
    }
    const bool use_tc = out && prefill_tc_supported(cfg->dtype, cfg->head_dim, cfg->rmsnorm, cfg->shared_kv);
    size_t need = 0;  // what this call uses: pooled entries without a cache, tensor-core scratch with an output
    if (!cache_out)
        need += align256((size_t)batch * cfg->n_kv_heads * NB * cfg->head_dim * esize_of(cfg->dtype)) *
                (cfg->shared_kv ? 1 : 2);
    if (use_tc) need += align256(prefill_tc_scratch_bytes(batch, T, cfg->n_kv_heads, cfg->rope_dims, cfg->block_m));
    if (workspace_bytes < need) return LBCA_ERR_CAPACITY;
    if (need > 0 && !workspace) return LBCA_ERR_ARG;
    if (out && !use_tc && !prefill_simt_supported(cfg->head_dim)) return LBCA_ERR_UNSUPPORTED;
    LBCA_TRY(check_device());
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    // 1. pool every complete block of K and V (and the open block's state)
    void* pk = cache_out ? cache_out->pooled_k : workspace;
    void* pv = nullptr;
    if (!cfg->shared_kv) {
        const size_t one = (size_t)batch * cfg->n_kv_heads * NB * cfg->head_dim * esize_of(cfg->dtype);
        pv = cache_out ? cache_out->pooled_v : static_cast<char*>(workspace) + align256(one);
    }
    const int stride = cache_out ? cache_out->max_blocks : NB;
    size_t pooled_bytes = 0;
    if (!cache_out) {
        const size_t one = (size_t)batch * cfg->n_kv_heads * NB * cfg->head_dim * esize_of(cfg->dtype);
        pooled_bytes = align256(one) * (cfg->shared_kv ? 1 : 2);
    }
    char* tc_scratch = static_cast<char*>(workspace) + pooled_bytes;
    PrefillArgs pa{};
    pa.dtype = cfg->dtype;
    pa.q = q; pa.k = k; pa.v = v; pa.pooled_k = pk; pa.pooled_v = cfg->shared_kv ? pk : pv;
    pa.pool_stride = stride; pa.sink = sink; pa.gamma_q = gamma_q; pa.gamma_kv = gamma_kv; pa.out = out;
    pa.B = batch; pa.T = T; pa.Hq = cfg->n_q_heads; pa.G = cfg->n_kv_heads; pa.D = cfg->head_dim;
    pa.m = m; pa.w = cfg->n_win; pa.rho = cfg->rope_dims; pa.rmsnorm = cfg->rmsnorm;
    pa.shared = cfg->shared_kv; pa.eps = cfg->rms_eps; pa.scale = scale_of(cfg); pa.rope_step = rope_step_of(cfg);
    pa.t_off = 0; pa.s_off = 0; pa.T_raw = T;
    // the tensor-core path: cos/sin table first, so that the pool pass can leave
    // fp16 copies of the raw keys (rotated) and values as it streams them
    if (use_tc) LBCA_TRY(cuda_status(launch_prefill_tc_table(pa, tc_scratch, s)));
    const PrefillRawF16 raw16 = use_tc ? prefill_tc_raw_f16(pa, tc_scratch) : PrefillRawF16{nullptr, nullptr, nullptr};
    {   // both series (or the shared entries) in one launch
        PoolArgs a{};
        a.dtype = cfg->dtype;
        a.nser = cfg->shared_kv ? 1 : 2;
        for (int series = 0; series < a.nser; ++series) {
            PoolSeries& sr = a.ser[series];
            sr.x = series ? v : k; sr.z = series ? zv : zk; sr.bpos = series ? b_pos_v : b_pos_k;
            sr.gamma = series ? nullptr : gamma_kv;
            sr.out = series ? pv : pk;
            sr.key = series == 0; sr.state_series = series;
            if (use_tc) {
                // the tensor-core MMAs read dense fp16 copies of the pooled keys and values, [B, G, NB, D]
                sr.out_f16 = tc_scratch + (series == 0
                                               ? prefill_tc_pooled_f16_offset(batch, T, cfg->n_kv_heads, cfg->rope_dims)
                                               : prefill_tc_pooled_v_f16_offset(batch, T, cfg->n_kv_heads,
                                                                                cfg->rope_dims, m));
                sr.raw_f16 = series == 0 ? raw16.keys : raw16.vals;
            }
        }
        a.out_blocks = stride; a.blk_off = 0; a.out_f16_blocks = NB;
        a.B = batch; a.T = T; a.G = cfg->n_kv_heads; a.D = cfg->head_dim; a.m = m; a.pos0 = 0;
        a.rmsnorm = cfg->rmsnorm; a.rho = cfg->rope_dims;
        a.rope_step = rope_step_of(cfg); a.eps = cfg->rms_eps;
        a.state = cache_out ? cache_out->pool_state : nullptr;
        a.S = cfg->shared_kv ? 1 : 2;
        a.tab = use_tc ? raw16.tab : nullptr;
        a.status = d_status;
        LBCA_TRY(cuda_status(launch_pool(a, s)));
    }
    // 2. the raw window and the lengths, so decode can continue from T
    if (cache_out) {
        RingFillArgs r{};
        r.dtype = cfg->dtype;
        r.k = k; r.v = v; r.gamma = gamma_kv;
        r.ring_k = cache_out->ring_k; r.ring_v = cache_out->ring_v; r.seq_lens = cache_out->seq_lens;
        r.B = batch; r.T = T; r.G = cfg->n_kv_heads; r.D = cfg->head_dim; r.R = cache_out->ring_slots;
        r.n = T < r.R ? T : r.R;
        r.rmsnorm = cfg->rmsnorm; r.rho = cfg->rope_dims; r.rope_step = rope_step_of(cfg); r.eps = cfg->rms_eps;
        LBCA_TRY(cuda_status(launch_ring_fill(r, s)));
    }
    // 3. attention
    if (out) {
        if (use_tc) {
            LBCA_TRY(cuda_status(launch_prefill_tc(pa, tc_scratch, d_status, s)));
        } else {
            LBCA_TRY(cuda_status(launch_prefill_simt(pa, s)));
        }
    }
    return LBCA_OK;
}

// ---- decode without a caller-provided workspace ---------------------------------------
// For callers that cannot allocate device memory (see lbca_decode_noalloc in the
// header).  The split partials and merge counters live in this file-scope
// device array instead of a caller workspace.  Every GPU that loads the library
// holds it until the process exits, so it is kept to LBCA_NOALLOC_SCRATCH_BYTES.
static __device__ __align__(256) unsigned char g_decode_scratch[LBCA_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_scratch_mu;
void* g_scratch_addr[64];  // device address of g_decode_scratch, per device ordinal

// In host code `g_decode_scratch` names a host-side shadow, not device memory;
// the device address is looked up once per device, with that device current.
lbca_status scratch_for_current_device(void** addr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LBCA_ERR_CUDA;
    if (dev < 0 || dev >= 64) return LBCA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return LBCA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return LBCA_OK;
}

}  // namespace

lbca_status lbca_decode_noalloc(const lbca_config* cfg, const void* q, const lbca_cache* cache,
                                const float* sink, const void* gamma_q, const void* gamma_kv, int32_t max_ctx,
                                void* out, int32_t* d_status, lbca_stream_t stream) {
    LBCA_TRY(check_cfg(cfg));
    LBCA_TRY(check_cache(cfg, cache));
    if (!q || !out) return LBCA_ERR_ARG;
    if (!al16(q) || !al16(out) || !al16n(gamma_q) || !al16n(gamma_kv) || !al16n(sink)) return LBCA_ERR_ALIGN;
    if (max_ctx <= 0) {
        const long long cap = (long long)cache->max_blocks * cfg->block_m + cache->ring_slots;
        max_ctx = cap > INT32_MAX ? INT32_MAX : (int32_t)(cap < 1 ? 1 : cap);
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the tensor-core kernel of the shared-entry form merges inside its cluster
    // and needs no scratch at all: no capacity check, no counters to clear
    if (mqa_tc_shape_ok(cfg->dtype, cache->batch, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim, cfg->block_m,
                        cfg->n_win, cfg->shared_kv, max_ctx)) {
        LBCA_TRY(check_device());
        DecodeArgs a = decode_args(cfg, q, cache, sink, gamma_q, gamma_kv, out, d_status);
        const MqaTcPlan tc = plan_decode_mqa_tc(cfg->dtype, a.B, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim,
                                                cfg->block_m, cfg->n_win, cfg->shared_kv, max_ctx);
        if (tc.cs > 0) {
            a.tc_cs = tc.cs;
            a.chunk = tc.rows;
            return cuda_status(launch_decode_mqa_tc(a, s));
        }
    }
    DecodePlan p = plan_decode(cfg->dtype, cache->batch, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim,
                               cfg->block_m, cfg->n_win, cfg->shared_kv, max_ctx);
    if (!p.ok) return LBCA_ERR_UNSUPPORTED;
    if (decode_workspace_bytes(p) > (size_t)LBCA_NOALLOC_SCRATCH_BYTES) return LBCA_ERR_CAPACITY;
    LBCA_TRY(check_device());
    void* scratch = nullptr;
    LBCA_TRY(scratch_for_current_device(&scratch));
    char* ws = static_cast<char*>(scratch);
    const size_t ctr_off = align256(p.part_o_elems * 4) + align256(p.part_ml_elems * 4);
    // the scratch keeps whatever the previous call left: the merge counters must start at zero
    if (cudaMemsetAsync(ws + ctr_off, 0, p.counter_elems * 4, s) != cudaSuccess) return LBCA_ERR_CUDA;
    DecodeArgs a = decode_args(cfg, q, cache, sink, gamma_q, gamma_kv, out, d_status);
    a.part_o = reinterpret_cast<float*>(ws);
    a.part_ml = reinterpret_cast<float*>(ws + align256(p.part_o_elems * 4));
    a.counters = reinterpret_cast<uint32_t*>(ws + ctr_off);
    a.n_split = p.n_split; a.chunk = p.chunk; a.heads_per_cta = p.heads_per_cta;
    return cuda_status(launch_decode(a, s));
}

lbca_status lbca_decode_sparse(const lbca_config* cfg, const void* q, const lbca_cache* cache, const int32_t* sel,
                               int32_t top_k, const float* sink, const void* gamma_q, const void* gamma_kv, void* out,
                               int32_t* d_status, lbca_stream_t stream) {
    LBCA_TRY(check_cfg(cfg));
    LBCA_TRY(check_cache(cfg, cache));
    if (!q || !out || !sel || top_k < 1) return LBCA_ERR_ARG;
    if (!al16(q) || !al16(out) || !al16n(gamma_q) || !al16n(gamma_kv) || !al16n(sink)) return LBCA_ERR_ALIGN;
    if (!cfg->shared_kv) return LBCA_ERR_UNSUPPORTED;
    if (cache->ring_slots < cfg->n_win) return LBCA_ERR_CAPACITY;
    const MqaTcPlan tc = plan_decode_mqa_tc_vis(cfg->dtype, cache->batch, cfg->n_q_heads, cfg->n_kv_heads,
                                                cfg->head_dim, cfg->shared_kv, (long long)top_k + cfg->n_win);
    if (tc.cs == 0) return cache->batch == 0 ? LBCA_OK : LBCA_ERR_UNSUPPORTED;
    LBCA_TRY(check_device());
    DecodeArgs a = decode_args(cfg, q, cache, sink, gamma_q, gamma_kv, out, d_status);
    a.sel = sel; a.sel_k = top_k;
    a.tc_cs = tc.cs; a.chunk = tc.rows;
    return cuda_status(launch_decode_mqa_tc(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t lbca_prefill_backward_workspace_bytes(const lbca_config* cfg, int32_t batch, int32_t T) {
    if (check_cfg(cfg) != LBCA_OK || batch < 0 || T < 0) return (size_t)-1;
    return align256(backward_scratch_floats(cfg->shared_kv ? 1 : 2, batch, T, cfg->n_q_heads, cfg->n_kv_heads,
                                            cfg->head_dim, cfg->block_m) * 4) + 256 * 10;
}

lbca_status lbca_prefill_backward(const lbca_config* cfg, const void* q, const void* k, const void* v, const void* zk,
                                  const void* zv, const void* b_pos_k, const void* b_pos_v, const float* sink,
                                  const void* gamma_q, const void* gamma_kv, const void* dout, int32_t batch, int32_t T, float* dq, float* dk, float* dv, float* dzk, float* dzv,
                                  float* db_pos_k, float* db_pos_v, float* dsink, void* workspace,
                                  size_t workspace_bytes, lbca_stream_t stream) {
    LBCA_TRY(check_cfg(cfg));
    if (batch < 0 || T < 0) return LBCA_ERR_ARG;
    const bool any = batch > 0 && T > 0;
    LBCA_TRY(check_kv(cfg, k, v, zk, zv, b_pos_k, b_pos_v, any));
    if (any && (!q || !dout || !dq || !dk || !dzk || !db_pos_k || !workspace)) return LBCA_ERR_ARG;
    if (any && !cfg->shared_kv && (!dv || !dzv || !db_pos_v)) return LBCA_ERR_ARG;
    if (any && sink && !dsink) return LBCA_ERR_ARG;
    if (!al16n(q) || !al16n(dout) || !al16n(workspace) || !al16n(gamma_q) || !al16n(gamma_kv))
        return LBCA_ERR_ALIGN;
    if (!backward_supported(cfg->head_dim)) return LBCA_ERR_UNSUPPORTED;
    if (workspace_bytes < lbca_prefill_backward_workspace_bytes(cfg, batch, T)) return LBCA_ERR_CAPACITY;
    if (!any) return LBCA_OK;
    LBCA_TRY(check_device());
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    BwdArgs a{};
    a.dtype = cfg->dtype;
    a.q = q; a.k = k; a.v = v; a.zk = zk; a.zv = zv; a.bpk = b_pos_k; a.bpv = b_pos_v; a.sink = sink;
    a.gamma_q = gamma_q; a.gamma_kv = gamma_kv; a.dout = dout;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dzk = dzk; a.dzv = dzv; a.dbk = db_pos_k; a.dbv = db_pos_v; a.dsink = dsink;
    a.B = batch; a.T = T; a.Hq = cfg->n_q_heads; a.G = cfg->n_kv_heads; a.D = cfg->head_dim; a.m = cfg->block_m;
    a.w = cfg->n_win; a.rho = cfg->rope_dims; a.rmsnorm = cfg->rmsnorm; a.shared = cfg->shared_kv;
    a.S = cfg->shared_kv ? 1 : 2; a.NB = T / cfg->block_m;
    a.eps = cfg->rms_eps; a.scale = scale_of(cfg); a.rope_step = rope_step_of(cfg);
    const size_t pooled = (size_t)a.S * batch * a.NB * a.G * a.D, raw = (size_t)batch * T * a.G * a.D;
    const size_t rows = (size_t)batch * T * a.Hq;
    float* f = static_cast<float*>(workspace);
    auto take = [&](size_t n) { float* p = f; f += (n + 63) / 64 * 64; return p; };
    a.Ef = take(pooled); a.dE = take(pooled); a.Pk = take((size_t)batch * a.NB * a.G * a.D);
    a.Kf = take(raw); a.dKf = take(raw); a.vf = a.shared ? nullptr : take(raw);
    a.qf = take(rows * a.D); a.dof = take(rows * a.D); a.lse = take(rows); a.dsum = take(rows);
    // the gradients that are accumulated, or written for complete blocks only, start at zero
    const size_t gd = (size_t)a.G * a.D;
    if (cudaMemsetAsync(dzk, 0, raw * 4, s) != cudaSuccess ||
        cudaMemsetAsync(db_pos_k, 0, (size_t)a.m * gd * 4, s) != cudaSuccess)
        return LBCA_ERR_CUDA;
    if (!cfg->shared_kv && (cudaMemsetAsync(dzv, 0, raw * 4, s) != cudaSuccess ||
                            cudaMemsetAsync(db_pos_v, 0, (size_t)a.m * gd * 4, s) != cudaSuccess))
        return LBCA_ERR_CUDA;
    if (sink && cudaMemsetAsync(dsink, 0, (size_t)a.Hq * 4, s) != cudaSuccess) return LBCA_ERR_CUDA;
    return cuda_status(launch_backward(a, s));
}

lbca_status lbca_prefill_rows(const lbca_config* cfg, const void* q, int32_t row0, int32_t n_rows, const void* k,
                              const void* v, int32_t raw0, int32_t n_raw, const float* pooled_k, const float* pooled_v,
                              int32_t pool_stride, const float* sink, const void* gamma_q, const void* gamma_kv,
                              int32_t batch, void* out, lbca_stream_t stream) {
    LBCA_TRY(check_cfg(cfg));
    if (batch < 0 || n_rows < 0 || n_raw < 0 || row0 < 0 || raw0 < 0 || pool_stride < 0) return LBCA_ERR_ARG;
    if (batch == 0 || n_rows == 0) return LBCA_OK;
    if (!q || !out || !k || (!cfg->shared_kv && !v) || (cfg->shared_kv && (v || pooled_v))) return LBCA_ERR_ARG;
    const int m = cfg->block_m, w = cfg->n_win;
    const long long last = (long long)row0 + n_rows;   // one past the last row
    const long long Plast = last - w > 0 ? (last - w) / m : 0;
    const long long Pfirst = (long long)row0 + 1 - w > 0 ? ((long long)row0 + 1 - w) / m : 0;
    // the raw rows must end at the last query and reach back to the first row's window
    if ((long long)raw0 + n_raw != last || raw0 > Pfirst * m) return LBCA_ERR_ARG;
    if (Plast > pool_stride || (Plast > 0 && (!pooled_k || (!cfg->shared_kv && !pooled_v)))) return LBCA_ERR_ARG;
    if (!al16(q) || !al16(out) || !al16(k) || !al16n(v) || !al16n(pooled_k) || !al16n(pooled_v) || !al16n(sink) ||
        !al16n(gamma_q) || !al16n(gamma_kv))
        return LBCA_ERR_ALIGN;
    if (!prefill_simt_supported(cfg->head_dim)) return LBCA_ERR_UNSUPPORTED;
    LBCA_TRY(check_device());
    PrefillArgs pa{};
    pa.dtype = cfg->dtype;
    pa.q = q; pa.k = k; pa.v = v; pa.pooled_k = pooled_k; pa.pooled_v = cfg->shared_kv ? pooled_k : pooled_v;
    pa.pool_stride = pool_stride; pa.pooled_f32 = 1; pa.sink = sink; pa.gamma_q = gamma_q; pa.gamma_kv = gamma_kv; pa.out = out;
    pa.B = batch; pa.T = n_rows; pa.Hq = cfg->n_q_heads; pa.G = cfg->n_kv_heads; pa.D = cfg->head_dim;
    pa.m = m; pa.w = w; pa.rho = cfg->rope_dims; pa.rmsnorm = cfg->rmsnorm; pa.shared = cfg->shared_kv;
    pa.eps = cfg->rms_eps; pa.scale = scale_of(cfg); pa.rope_step = rope_step_of(cfg);
    pa.t_off = row0; pa.s_off = raw0; pa.T_raw = n_raw;
    return cuda_status(launch_prefill_simt(pa, reinterpret_cast<cudaStream_t>(stream)));
}

size_t lbca_indexer_workspace_bytes(int32_t batch, int32_t max_blocks) {
    if (batch < 0 || max_blocks < 0) return 0;
    return align256((size_t)batch * max_blocks * 4);
}

lbca_status lbca_indexer_topk(int32_t batch, int32_t n_heads, int32_t head_dim, int32_t block_m, int32_t top_k,
                              const void* q_idx, const float* w_idx, const void* k_idx, int32_t max_blocks,
                              const int32_t* seq_lens, int32_t* sel, float* sel_scores, void* workspace,
                              size_t workspace_bytes, int32_t* d_status, lbca_stream_t stream) {
    if (batch < 0 || block_m < 1 || top_k < 1 || max_blocks < 0) return LBCA_ERR_ARG;
    if (!q_idx || !w_idx || !k_idx || !seq_lens || !sel || !workspace) return LBCA_ERR_ARG;
    if (!indexer_shape_ok(n_heads, head_dim)) return LBCA_ERR_UNSUPPORTED;
    if (!al16(q_idx) || !al16(k_idx) || !al16(workspace)) return LBCA_ERR_ALIGN;
    if (workspace_bytes < lbca_indexer_workspace_bytes(batch, max_blocks)) return LBCA_ERR_CAPACITY;
    LBCA_TRY(check_device());
    IndexerArgs a{};
    a.q_idx = q_idx; a.w_idx = w_idx; a.k_idx = k_idx; a.seq_lens = seq_lens;
    a.scores = static_cast<float*>(workspace); a.sel = sel; a.sel_scores = sel_scores; a.status = d_status;
    a.B = batch; a.HI = n_heads; a.DI = head_dim; a.m = block_m; a.max_blocks = max_blocks; a.top_k = top_k;
    return cuda_status(launch_indexer_topk(a, reinterpret_cast<cudaStream_t>(stream)));
}

const char* lbca_status_string(lbca_status status) {
    switch (status) {
        case LBCA_OK: return "ok";
        case LBCA_ERR_ARG: return "invalid argument";
        case LBCA_ERR_UNSUPPORTED: return "unsupported device or shape";
        case LBCA_ERR_CAPACITY: return "cache or workspace too small";
        case LBCA_ERR_CUDA: return "CUDA error";
        case LBCA_ERR_TIMEOUT: return "bounded device wait timed out";
        case LBCA_ERR_ALIGN: return "pointer not 16-byte aligned";
        default: return "unknown status";
    }
}

}  // extern "C"
