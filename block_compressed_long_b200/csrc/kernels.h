// kernels.h -- launch interfaces between the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "lbca.h"

namespace lbca {

// One pooled series of a pool launch.
struct PoolSeries {
    const void* x;         // [B, T, G, D]
    const void* z;         // [B, T, G, D]
    const void* bpos;      // [m, G*D]
    const void* gamma;     // [D] or null (key series with RMSNorm)
    void* out;             // [B, G, out_blocks, D]; block j at blk_off + j (or null)
    float* out_f32;        // optional f32 entries, same layout as out
    void* out_f16;         // optional fp16 copy [B, G, out_f16_blocks, D] (bf16 input only)
    // optional fp16 copy of every token of each complete block, [B, T, G, D]
    // (bf16 input only); key series rotated at their position s with cos/sin
    // from PoolArgs::tab ([rho/2][T], pair-major)
    void* raw_f16;
    int key;               // 1: key series (RMSNorm when on, RoPE at the block start)
    int state_series;      // index of this series in the pooling state
    // dual overlapped pooling (CSA form): the b-series [B, T, G, D] and its
    // bias [m, G*D]; entry j pools block j of (x, z) and block j - 1 of
    // (xb, zb) under one softmax.  Null for single-series pooling.
    const void* xb;
    const void* zb;
    const void* bposb;
};
// Pool complete blocks of one or two series in one launch (and optionally
// record the open block's running state).
struct PoolArgs {
    int dtype;
    PoolSeries ser[2];
    int nser;
    int out_blocks, blk_off, out_f16_blocks;
    int B, T, G, D, m;
    int64_t pos0;          // absolute position of token 0 of x
    int rmsnorm, rho;
    double rope_step;  // theta^(-2/rho)
    float eps;
    float* state;          // [B, S, 3, G, D] or null: running state of the partial block
    int S;
    const float2* tab;
    // device status word for the fp16 copies: a value beyond the fp16 range
    // sets LBCA_ERR_UNSUPPORTED (nullable)
    int32_t* status;
    // launch geometry (set by launch_pool): blocks per series and sequence,
    // head slices
    int nblk, gz;
    int dual;              // 1: every series is pooled in the dual overlapped form
};
cudaError_t launch_pool(const PoolArgs& a, cudaStream_t s);

// Write finalised raw keys / raw values of tokens [T - n, T) into the ring and
// set seq_lens = T.
struct RingFillArgs {
    int dtype;
    const void* k;         // [B, T, G, D]
    const void* v;         // [B, T, G, D] or null (shared form)
    const void* gamma;
    void* ring_k;          // [B, G, R, D]
    void* ring_v;
    int32_t* seq_lens;
    int B, T, G, D, R, n;
    int rmsnorm, rho;
    double rope_step;  // theta^(-2/rho)
    float eps;
};
cudaError_t launch_ring_fill(const RingFillArgs& a, cudaStream_t s);

struct AppendArgs {
    int dtype;
    const void* k; const void* v; const void* zk; const void* zv;  // [B, G, D]
    const void* bpk; const void* bpv;                              // [m, G*D]
    const void* gamma;
    void* pooled_k; void* pooled_v;                                // [B, G, max_blocks, D]
    void* ring_k; void* ring_v;                                    // [B, G, R, D]
    float* state;                                                  // [B, S, 3, G, D]
    int32_t* seq_lens;
    int32_t* status;
    int B, G, D, m, R, max_blocks, S;
    int rmsnorm, rho;
    double rope_step;  // theta^(-2/rho)
    float eps;
};
cudaError_t launch_append(const AppendArgs& a, cudaStream_t s);

struct DecodeArgs {
    int dtype;
    const void* q;                                   // [B, Hq, D]
    const void* pooled_k; const void* pooled_v;      // [B, G, max_blocks, D]
    const void* ring_k; const void* ring_v;          // [B, G, R, D]
    const int32_t* seq_lens;
    const float* sink;
    const void* gamma_q;
    void* out;                                       // [B, Hq, D]
    float* part_o;                                   // [B, Hq, n_split, D]
    float* part_ml;                                  // [B, Hq, n_split, 2]
    uint32_t* counters;                              // [B, Hq / heads_per_cta]
    int32_t* status;
    int B, Hq, G, D, m, w, rho, rmsnorm, shared, max_blocks, R;
    int n_split, chunk, heads_per_cta;
    int tc_cs;         // tensor-core shared-entry path: CTAs per cluster (0 = CUDA-core path)
    float eps, scale;
    double rope_step;  // theta^(-2/rho)
    // Append fused into the tensor-core shared-entry kernel (app_k == nullptr:
    // none; one kv head only).  The new token [B, G, D] and its Z logits join
    // the cache first, then the query at the new length attends.
    const void* app_k; const void* app_z; const void* app_bp; const void* gamma_kv;
    void* ring_w; void* pooled_w;                    // the cache's ring_k / pooled_k, written
    float* state;                                    // [B, 1, 3, G, D]
    int32_t* lens_w;                                 // seq_lens, advanced by one
    // CSA form (tensor-core shared-entry decode only): the selected entries
    // [B, sel_k] (block indices, valid ones first) replace the pooled prefix,
    // and the raw window is the last n_win tokens; null: block-aligned partition
    const int32_t* sel;
    int sel_k;
    int pdl;           // launch with programmatic dependence on the preceding kernel (cache reads first)
};
// Chooses heads per CTA, chunk and split count for a decode call.
struct DecodePlan {
    int heads_per_cta, chunk, n_split;
    size_t part_o_elems, part_ml_elems, counter_elems;
    size_t smem_bytes;
    bool ok;
};
DecodePlan plan_decode(int dtype, int B, int Hq, int G, int D, int m, int w, int shared,
                       int max_ctx);
size_t decode_workspace_bytes(const DecodePlan& p);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);
// Tensor-core decode of the shared-entry form (bf16, 64 query heads per kv head,
// D in {256, 512}): CTAs per cluster (0 when the kernel does not apply) and
// entry rows per CTA.  Launch with DecodeArgs.tc_cs = cs and .chunk = rows.
struct MqaTcPlan {
    int cs, rows;
};
MqaTcPlan plan_decode_mqa_tc(int dtype, int B, int Hq, int G, int D, int m, int w, int shared, int max_ctx);
// The same plan for a visible list of at most max_vis entries (the CSA form:
// top_k selected entries plus n_win window tokens).
MqaTcPlan plan_decode_mqa_tc_vis(int dtype, int B, int Hq, int G, int D, int shared, long long max_vis);
// The shape tests of plan_decode_mqa_tc alone (host-only, no device query).
bool mqa_tc_shape_ok(int dtype, int B, int Hq, int G, int D, int m, int w, int shared, int max_ctx);
cudaError_t launch_decode_mqa_tc(const DecodeArgs& a, cudaStream_t s);

// One serving step (append + decode) in one cluster launch.
struct StepArgs {
    int dtype;
    const void* k; const void* v; const void* zk; const void* zv;  // [B, G, D] the new token
    const void* bpk; const void* bpv; const void* gamma_kv;
    const void* q; const float* sink; const void* gamma_q;         // q [B, Hq, D]
    void* out;                                                     // [B, Hq, D]
    void* pooled_k; void* pooled_v; void* ring_k; void* ring_v;
    float* state; int32_t* seq_lens;
    uint32_t* arrive;                                              // [B] arrival counters (zeroed)
    int32_t* status;
    int B, Hq, G, D, m, w, rho, rmsnorm, shared, max_blocks, R, S;
    int CS, SE, heads_per_cta;
    float eps, scale;
    double rope_step;  // theta^(-2/rho)
    // persistent evenly-split form (decode_flat.cu): arrive is one grid-wide counter
    float* part_o;                                                 // [segments][maxc][R][D]
    float* part_ml;                                                // [segments][maxc][R][2]
    uint32_t* seg_count;                                           // [segments], zeroed
    int C, grid, maxc;
    uint64_t rope_f[128];  // persistent form: fixed-point turns per position of each RoPE pair (rope_turns)
    int pdl;               // launch with programmatic dependence on the preceding kernel (cache reads first)
};
struct StepPlan {
    int heads_per_cta, CS, SE;
    size_t arrive_elems, smem_bytes;
    bool ok;
    // persistent evenly-split form: chosen for large batches
    bool flat;
    int C, maxc;
    size_t seg_elems, part_o_elems, part_ml_elems;
};
StepPlan plan_step(int dtype, int B, int Hq, int G, int D, int m, int w, int shared, int max_ctx);
size_t step_workspace_bytes(const StepPlan& p);
cudaError_t launch_decode_step(const StepArgs& a, cudaStream_t s);
size_t flat_smem_bytes(int dtype, int B, int D, int R, int C, int shared);
cudaError_t launch_decode_flat(const StepArgs& a, cudaStream_t s);
// CTAs of the persistent grid on the current device (every SM filled).
cudaError_t flat_grid(int* grid, int dtype, int D, int R, size_t smem);

// Lightning-indexer relevance and top-k selection (CSA form): one query per
// sequence, bf16 queries [B, HI, DI] and compressed keys [B, max_blocks, DI].
struct IndexerArgs {
    const void* q_idx; const float* w_idx; const void* k_idx; const int32_t* seq_lens;
    float* scores;                                   // [B, max_blocks] workspace
    int32_t* sel;                                    // [B, top_k]
    float* sel_scores;                               // [B, top_k] or null
    int32_t* status;
    int B, HI, DI, m, max_blocks, top_k;
};
bool indexer_shape_ok(int HI, int DI);
cudaError_t launch_indexer_topk(const IndexerArgs& a, cudaStream_t s);

// Backward of the prefill (pooling + attention): f32 gradients and scratch.
struct BwdArgs {
    int dtype;
    const void* q; const void* k; const void* v; const void* zk; const void* zv;
    const void* bpk; const void* bpv; const float* sink; const void* gamma_q; const void* gamma_kv;
    const void* dout;                                  // gradient of the forward's output [B, T, Hq, D]
    float* dq; float* dk; float* dv; float* dzk; float* dzv; float* dbk; float* dbv; float* dsink;
    // scratch: Ef, dE [S][B][NB][G][D]; Pk [B][NB][G][D]; Kf, dKf, vf [B][T][G][D];
    // qf, dof [B][T][Hq][D]; lse, dsum [B][T][Hq]
    float* Ef; float* dE; float* Pk; float* Kf; float* dKf; float* vf; float* qf; float* dof; float* lse;
    float* dsum;
    int B, T, Hq, G, D, m, w, rho, rmsnorm, shared, S, NB;
    float eps, scale;
    double rope_step;
};
bool backward_supported(int D);
size_t backward_scratch_floats(int S, int B, int T, int Hq, int G, int D, int m);
cudaError_t launch_backward(const BwdArgs& a, cudaStream_t s);

struct PrefillArgs {
    int dtype;
    const void* q;                                   // [B, T, Hq, D]
    const void* k; const void* v;                    // raw [B, T, G, D]
    const void* pooled_k; const void* pooled_v;      // [B, G, pool_stride, D]
    int pool_stride;
    int pooled_f32;                                  // 1: pooled entries are f32 (row-range form)
    const float* sink;
    const void* gamma_q; const void* gamma_kv;
    void* out;                                       // [B, T, Hq, D]
    int B, T, Hq, G, D, m, w, rho, rmsnorm, shared;
    float eps, scale;
    double rope_step;  // theta^(-2/rho)
    // row range (CUDA-core kernel): q / out rows at absolute positions t_off ..
    // t_off + T - 1; k / v hold T_raw rows from absolute position s_off
    // (the whole-sequence prefill: 0, 0, T)
    int t_off, s_off, T_raw;
};
cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s);
// Tensor-core prefill (bf16, D = 128, GQA form without RMSNorm); `scratch` holds
// prefill_tc_scratch_bytes (finalised raw keys and the RoPE table).
bool prefill_tc_supported(int dtype, int D, int rmsnorm, int shared);
size_t prefill_tc_scratch_bytes(int B, int T, int G, int rho, int m);
// where, inside that scratch, the pool pass leaves the fp16 copy of the pooled keys
size_t prefill_tc_pooled_f16_offset(int B, int T, int G, int rho);
size_t prefill_tc_pooled_v_f16_offset(int B, int T, int G, int rho, int m);
// The parts of that scratch the pool pass fills for the tensor-core kernel: fp16
// raw keys (rotated) and values of every complete block, from the cos/sin table.
struct PrefillRawF16 {
    void* keys; void* vals; const float2* tab;
};
PrefillRawF16 prefill_tc_raw_f16(const PrefillArgs& a, void* scratch);
// 1. the cos/sin table (before the pool pass); 2. the tail tokens past the last
// complete block, then the attention kernel (after it).
cudaError_t launch_prefill_tc_table(const PrefillArgs& a, void* scratch, cudaStream_t s);
cudaError_t launch_prefill_tc(const PrefillArgs& a, void* scratch, int32_t* status, cudaStream_t s);
bool prefill_simt_supported(int D);

}  // namespace lbca
