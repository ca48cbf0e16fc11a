/*
 * lbca.h -- C ABI of the B200 (sm_100a) block-compressed attention library.
 *
 * Block-compressed attention as in LBCA ("mSeek: learned KV-cache compression
 * in a 3B model", section "How LBCA works") and HCA ("HCA: Heavily Compressed
 * Attention", section "What is implemented"):
 *   - every complete, non-overlapping block of m raw tokens is pooled into one
 *     entry by a per-channel softmax over the block's positions of content
 *     logits Z plus a learnable positional bias B_pos (HCA page, Eqs 20-23);
 *   - a query attends, in one softmax, to every causally visible pooled entry
 *     plus an exact window of recent raw tokens, plus an optional attention
 *     sink logit (CSA page, "What is implemented": Eqs 18-19 and Eq 27);
 *   - key entries take RMSNorm (HCA form) and partial RoPE; pooled entries are
 *     rotated at their block-start position (CSA page, "Deviations from
 *     paper"); in the shared K=V form the output's RoPE dims are rotated by
 *     the negative query position (CSA page, "What is implemented").
 *
 * Visibility (the reading under which the mSeek README's cache figures come
 * out exactly): a query at 0-based position t sees L = t + 1 tokens, the
 * pooled entries j < P(L) = max(0, floor((L - n_win) / m)), and the raw
 * tokens s in [P(L) * m, t].  Blocks that are incomplete stay raw.
 *
 * Conventions shared by every entry point
 *   - All tensors are caller-owned, row-major, contiguous, and 16-byte
 *     aligned; the library never allocates device memory.  Pointers named
 *     "device" must be device (or managed) memory of the current device.
 *   - I/O tensors have the config's dtype (bf16 or f32); arithmetic is f32.
 *     Sinks are f32 in natural-log units.  gamma pointers are RMSNorm gains
 *     [D] in the I/O dtype, or NULL for a gain of one.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  The return value reports host-side validation and
 *     launch errors only; it never waits for the GPU.  Conditions found on the
 *     device are written to the optional device word `d_status` (an
 *     lbca_status; it is only ever set to a non-zero value, so zero it before
 *     the calls whose outcome you want to read).
 *   - Nothing aborts the process: bad arguments return LBCA_ERR_ARG before any
 *     CUDA call, a device other than sm_100 returns LBCA_ERR_UNSUPPORTED.
 */
#ifndef LBCA_H
#define LBCA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LBCA_API __attribute__((visibility("default")))
#else
#define LBCA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* lbca_stream_t; /* == cudaStream_t */

typedef enum {
    LBCA_OK = 0,
    LBCA_ERR_ARG = 1,         /* invalid argument (host-side check)            */
    LBCA_ERR_UNSUPPORTED = 2, /* device is not sm_100, or shape not supported  */
    LBCA_ERR_CAPACITY = 3,    /* cache or workspace too small for the request  */
    LBCA_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed          */
    LBCA_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up            */
    LBCA_ERR_ALIGN = 6        /* a pointer is not 16-byte aligned              */
} lbca_status;

typedef enum { LBCA_F32 = 0, LBCA_BF16 = 1 } lbca_dtype;

/* Which pooled series lbca_pool produces: keys are finalised (RMSNorm when
 * enabled, RoPE at the block start); values are stored as pooled.  In the
 * shared K=V form the single series is LBCA_KEY. */
typedef enum { LBCA_KEY = 0, LBCA_VALUE = 1 } lbca_series;

typedef struct {
    int32_t n_q_heads;     /* Hq >= 1                                                 */
    int32_t n_kv_heads;    /* G >= 1, Hq % G == 0; query head h uses kv head h/(Hq/G) */
    int32_t head_dim;      /* D: a multiple of 16 in [16, 512]                        */
    int32_t shared_kv;     /* 1: one entry serves as key and value (HCA MQA form)     */
    int32_t block_m;       /* m >= 1 raw tokens per pooled entry                      */
    int32_t n_win;         /* n_win >= 0 raw window                                   */
    int32_t rope_dims;     /* rho: RoPE on the last rho dims (even, <= D); 0 = off    */
    int32_t rmsnorm;       /* 1: RMSNorm on queries and key entries (pooled and raw)  */
    double  rope_theta;    /* base; pair k of the rotated dims turns by
                              pos * theta^(-2k/rho); consecutive pairs (2k, 2k+1)    */
    float   rms_eps;       /* RMSNorm epsilon: x / sqrt(mean(x^2) + eps) * gamma      */
    float   softmax_scale; /* <= 0 selects 1/sqrt(D)                                  */
    int32_t dtype;         /* lbca_dtype of every I/O tensor                         */
    int32_t reserved;      /* must be 0                                               */
} lbca_config;

/*
 * Decode-time cache of B sequences (caller-owned device memory; zero-filled
 * memory with seq_lens = 0 is an empty cache).  Written by lbca_prefill and
 * lbca_append, read by lbca_decode.
 *   pooled_k   [B, G, max_blocks, D] finalised pooled key entries (shared form:
 *              the entries, used as key and value)
 *   pooled_v   [B, G, max_blocks, D] pooled values; NULL in the shared form
 *   ring_k     [B, G, ring_slots, D] raw window; token s in slot s % ring_slots.  GQA
 *              form: the finalised keys (RMSNorm when enabled, RoPE at s).  Shared
 *              form: the raw entries C exactly as appended, finalised (RMSNorm,
 *              RoPE at s) in f32 by the decode kernels when read -- there the
 *              row also serves as the value, so it is not rounded a second time
 *   ring_v     [B, G, ring_slots, D] raw values; NULL in the shared form
 *   pool_state [B, S, 3, G, D] f32 running (max, sum, weighted sum) of the
 *              open block's pooling softmax, S = 2 (K then V) or 1 (shared)
 *   seq_lens   [B] int32 tokens cached per sequence
 * ring_slots must be >= lbca_ring_slots(cfg).
 */
typedef struct {
    void*    pooled_k;
    void*    pooled_v;
    void*    ring_k;
    void*    ring_v;
    float*   pool_state;
    int32_t* seq_lens;
    int32_t  batch;
    int32_t  max_blocks;
    int32_t  ring_slots;
    int32_t  flags;        /* 0, or LBCA_CACHE_OVERLAP_PREV */
} lbca_cache;

/* lbca_cache.flags: the one-launch serving steps (lbca_decode_step in its fused
 * forms) may start before the preceding work on the stream has finished and
 * read this cache (lengths, pooling state, entries, window) while it drains
 * (programmatic dependent launch); the step's own inputs -- the query and the
 * new token -- are read, and anything is written, only once that work has
 * completed.  Set it only when the preceding work does not write this cache:
 * in a model, the other layers' kernels that run between two steps of this
 * layer.  Two steps of the same cache back to back must not set it. */
#define LBCA_CACHE_OVERLAP_PREV 1

/* Minimum ring slots: m * ceil((n_win + m - 1) / m), the most raw tokens a
 * query can see rounded up to whole blocks.  -1 on an invalid config. */
LBCA_API int32_t lbca_ring_slots(const lbca_config* cfg);

/* f32 elements of lbca_cache.pool_state for `batch` sequences; 0 on error. */
LBCA_API size_t lbca_pool_state_elems(const lbca_config* cfg, int32_t batch);

/* Bytes of `workspace` lbca_decode needs for `batch` sequences whose lengths
 * never exceed max_ctx; 0 on error.  The workspace must be zero-filled before
 * its first use; lbca_decode leaves it zero-filled again. */
LBCA_API size_t lbca_decode_workspace_bytes(const lbca_config* cfg, int32_t batch, int32_t max_ctx);

/* Bytes of `workspace` lbca_prefill needs (0 when a cache receives the
 * pooled entries); (size_t)-1 on error. */
LBCA_API size_t lbca_prefill_workspace_bytes(const lbca_config* cfg, int32_t batch, int32_t T,
                                    int32_t has_cache);

/*
 * lbca_pool -- pool the floor(T/m) complete blocks of one series.
 * (HCA page, "What is implemented": single-series pooling, Eqs 20-23; mSeek
 * README, "How LBCA works", steps 2-3; entry RoPE at block starts: CSA page,
 * "Deviations from paper".)
 *   x, z      device [B, T, G, D] raw values and content logits
 *   b_pos     device [m, G*D] positional bias, indexed by in-block offset
 *   gamma     device [D] RMSNorm gain (key series with rmsnorm) or NULL
 *   pos0      absolute position of x's first token; a multiple of m
 *   out       device [B, G, out_blocks, D]; block j of this call is written at
 *             index pos0/m + j, which must be < out_blocks
 * Per (block j, kv head g, channel c):
 *   w_i = softmax_i(Z[jm+i, g, c] + B_pos[i, g*D + c]),  out = sum_i w_i X[jm+i, g, c],
 * then, for LBCA_KEY: RMSNorm (when enabled) and RoPE at position pos0 + j*m.
 * Errors: LBCA_ERR_ARG (null/bad sizes, pos0 % m != 0, out_blocks too small),
 * LBCA_ERR_ALIGN, LBCA_ERR_UNSUPPORTED, LBCA_ERR_CUDA.
 */
LBCA_API lbca_status lbca_pool(const lbca_config* cfg, int32_t series, const void* x, const void* z,
                      const void* b_pos, const void* gamma, int32_t batch, int32_t T,
                      int32_t pos0, void* out, int32_t out_blocks, lbca_stream_t stream);

/*
 * lbca_pool_kv -- lbca_pool of both series of the GQA form in one launch: the
 * keys (k, zk, b_pos_k, gamma_kv: RMSNorm when enabled and RoPE at each block
 * start) into pooled_k, the values (v, zv, b_pos_v, pooled as is) into
 * pooled_v.  Each series' arguments mean what they mean in lbca_pool; the
 * entries equal those of two lbca_pool calls bit for bit (HCA page, "What is
 * implemented", Eqs 20-23; mSeek README, "How LBCA works", steps 2-3).
 * Errors: as lbca_pool; LBCA_ERR_ARG also for the shared form (no value series).
 */
LBCA_API lbca_status lbca_pool_kv(const lbca_config* cfg, const void* k, const void* v, const void* zk,
                         const void* zv, const void* b_pos_k, const void* b_pos_v,
                         const void* gamma_kv, int32_t batch, int32_t T, int32_t pos0,
                         void* pooled_k, void* pooled_v, int32_t out_blocks, lbca_stream_t stream);

/*
 * lbca_pool_f32 -- lbca_pool with the entries written in f32 (out: device
 * [B, G, out_blocks, D] float), unrounded: the exchange format of a
 * context-parallel prefill, whose ranks all-gather their pooled entries and
 * read them with lbca_prefill_rows at the precision the single-GPU prefill
 * keeps them.  Same arguments, arithmetic and errors as lbca_pool.
 */
LBCA_API lbca_status lbca_pool_f32(const lbca_config* cfg, int32_t series, const void* x, const void* z,
                                   const void* b_pos, const void* gamma, int32_t batch, int32_t T,
                                   int32_t pos0, float* out, int32_t out_blocks, lbca_stream_t stream);

/*
 * lbca_pool_dual -- dual overlapped pooling of the floor(T/m) complete blocks
 * (the CSA form; CSA page, "What is implemented": dual overlapped
 * compression, Eqs 9-12; entry RoPE at block starts: "Deviations from paper").
 *   xa, za      device [B, T, G, D] a-series raw values and content logits
 *   xb, zb      device [B, T, G, D] b-series raw values and content logits
 *   b_pos_a/_b  device [m, G*D] positional biases of the two series
 *   gamma       device [D] RMSNorm gain (key series with rmsnorm) or NULL
 *   out         device [B, G, out_blocks, D]; entry j at index j < out_blocks
 * Per (entry j, kv head g, channel c), ONE softmax over the 2m logits of block
 * j of the a-series and block j - 1 of the b-series (entry 0: its m a-series
 * logits alone) weights the matching raw values:
 *   out_j = sum_r w_a[r] xa[j m + r] + sum_r w_b[r] xb[(j - 1) m + r],
 * then, for LBCA_KEY: RMSNorm (when enabled) and RoPE at position j m.  Each
 * token of each series is read once.  The CSA form's indexer keys are pooled
 * the same way with their own series (LBCA_VALUE: no finalisation).
 * Errors: LBCA_ERR_ARG (null or bad sizes, out_blocks < T / m),
 * LBCA_ERR_ALIGN, LBCA_ERR_UNSUPPORTED, LBCA_ERR_CUDA.
 */
LBCA_API lbca_status lbca_pool_dual(const lbca_config* cfg, int32_t series, const void* xa, const void* za,
                                    const void* xb, const void* zb, const void* b_pos_a, const void* b_pos_b,
                                    const void* gamma, int32_t batch, int32_t T, void* out, int32_t out_blocks,
                                    lbca_stream_t stream);

/*
 * lbca_append -- add one raw token to every sequence of the cache.
 * (mSeek README, repository layout: generation through the LBCA cache; "How
 * LBCA works", step 5: incomplete blocks stay raw.)
 *   k, v, zk, zv  device [B, G, D] the token's key, value and their content
 *                 logits (shared form: k = C, zk = Z, v = zv = NULL)
 *   b_pos_k/_v    device [m, G*D] positional biases (b_pos_v NULL when shared)
 *   gamma_kv      device [D] key RMSNorm gain or NULL
 * For sequence b the token's position is p = seq_lens[b]: its finalised key
 * (RMSNorm, RoPE at p) and raw value go to ring slot p % ring_slots, the
 * running pooling softmax of block p/m is updated, and when p % m == m - 1 the
 * block's entry is finalised into pooled_k/v[b, :, p/m].  seq_lens[b] becomes
 * p + 1.  If block p/m >= max_blocks the entry is dropped and d_status is set
 * to LBCA_ERR_CAPACITY.
 */
LBCA_API lbca_status lbca_append(const lbca_config* cfg, const void* k, const void* v, const void* zk,
                        const void* zv, const void* b_pos_k, const void* b_pos_v,
                        const void* gamma_kv, const lbca_cache* cache, int32_t* d_status,
                        lbca_stream_t stream);

/*
 * lbca_decode -- attention of one query per sequence at its last position.
 * (mSeek README, "How LBCA works", step 4; HCA page, "What is implemented":
 * every compressed entry the query may causally see, attended densely with
 * the raw window, one key/value entry shared by all query heads, RMSNorm,
 * RoPE on part of the dims and a sink; CSA page, "What is implemented":
 * Eqs 18-19, Eq 27, outputs turned back by -t.)
 *   q          device [B, Hq, D] queries; sequence b's query sits at position
 *              t = seq_lens[b] - 1 (call lbca_append for the token first)
 *   sink       device [Hq] f32 sink logits or NULL
 *   gamma_q    device [D] query RMSNorm gain or NULL
 *   gamma_kv   device [D] key RMSNorm gain or NULL: the one given to lbca_append
 *              and lbca_prefill (the shared form finalises its raw window here)
 *   max_ctx    upper bound of seq_lens (sizes the split grid); <= 0 derives it
 *              from the cache capacity
 *   out        device [B, Hq, D]
 *   workspace  device, >= lbca_decode_workspace_bytes(cfg, B, max_ctx) bytes,
 *              zero-filled before first use (left zero-filled)
 * The visible entries are split into chunks processed by separate CTAs; the
 * last CTA of each (sequence, head group) merges the partial softmaxes.
 * A sequence with no tokens yields zeros.  A sequence longer than max_ctx sets
 * d_status to LBCA_ERR_CAPACITY (its output is then incomplete).  The
 * shared-entry form on the tensor cores (bf16, 64 query heads per kv head,
 * D 256 or 512) multiplies in fp16: an entry or query beyond the fp16 range
 * sets d_status to LBCA_ERR_UNSUPPORTED.
 * Calls that share a workspace must not overlap on the GPU.
 */
LBCA_API lbca_status lbca_decode(const lbca_config* cfg, const void* q, const lbca_cache* cache,
                        const float* sink, const void* gamma_q, const void* gamma_kv, int32_t max_ctx, void* out,
                        void* workspace, size_t workspace_bytes, int32_t* d_status,
                        lbca_stream_t stream);

/*
 * lbca_decode_step -- one serving step: lbca_append of the token (k, v, zk, zv)
 * followed by lbca_decode of q, in one launch where the shapes allow.
 * (mSeek README, repository layout: generation through the LBCA cache; "How
 * LBCA works", steps 2-5.)  Arguments as in lbca_append and lbca_decode;
 * `workspace` (zero-filled before first use, left zero-filled) must hold
 * lbca_decode_step_workspace_bytes(cfg, B, max_ctx) bytes.  In the GQA form
 * with n_win >= 1, D in {64, 128, 256} and up to 4 query heads per kv head per
 * CTA group, the step runs as one kernel (the appended token's block cannot be visible to
 * the same query, so appending and attending are independent): for a few
 * (sequence, head group) pairs a cluster kernel that splits each pair's
 * entries over the CTAs of a cluster, for many pairs (96 or more) a
 * persistent kernel whose CTAs each take an equal share of all the step's
 * entries, whatever the mix of context lengths.  The shared-entry form on
 * the tensor-core decode (bf16, 64 query heads per kv head, D in {256, 512})
 * with one kv head and n_win >= 1 also runs as one kernel: the CTA that holds
 * the newest visible row appends the token.  Other shapes run lbca_append
 * then lbca_decode.  Results equal those of the two calls.  A sequence longer
 * than max_ctx sets d_status to LBCA_ERR_CAPACITY.
 */
LBCA_API size_t lbca_decode_step_workspace_bytes(const lbca_config* cfg, int32_t batch, int32_t max_ctx);
/* Kernel launches one lbca_decode_step call makes for these shapes: 1 when the
 * step runs as one fused kernel, 2 when it runs lbca_append then lbca_decode,
 * -1 for an invalid configuration.  Host-only; needs no GPU. */
LBCA_API int32_t lbca_decode_step_launches(const lbca_config* cfg, int32_t batch, int32_t max_ctx);
/* Which form lbca_decode_step takes for these shapes (host-only; needs no GPU). */
typedef enum {
    LBCA_STEP_TWO_CALLS = 0,   /* lbca_append, then lbca_decode */
    LBCA_STEP_CLUSTER = 1,     /* one cluster kernel */
    LBCA_STEP_PERSISTENT = 2,  /* one persistent, evenly split kernel */
    LBCA_STEP_SHARED_TC = 3    /* one tensor-core shared-entry kernel, append fused */
} lbca_step_form;
/* Returns an lbca_step_form, or -1 for an invalid configuration. */
LBCA_API int32_t lbca_decode_step_form(const lbca_config* cfg, int32_t batch, int32_t max_ctx);
LBCA_API lbca_status lbca_decode_step(const lbca_config* cfg, const void* k, const void* v, const void* zk,
                                      const void* zv, const void* b_pos_k, const void* b_pos_v,
                                      const void* gamma_kv, const void* q, const lbca_cache* cache,
                                      const float* sink, const void* gamma_q, int32_t max_ctx, void* out,
                                      void* workspace, size_t workspace_bytes, int32_t* d_status,
                                      lbca_stream_t stream);

/*
 * lbca_prefill -- causal block-compressed attention over T tokens per sequence.
 * (mSeek README, "How LBCA works", steps 1-5; HCA page, "What is implemented";
 * CSA page, "What is implemented" and "Deviations from paper".)
 *   q            device [B, T, Hq, D]
 *   k, v, zk, zv device [B, T, G, D] (shared form: k = C, zk = Z, v = zv = NULL)
 *   b_pos_k/_v   device [m, G*D]
 *   sink         device [Hq] f32 or NULL; gamma_q, gamma_kv device [D] or NULL
 *   out          device [B, T, Hq, D], or NULL to only fill `cache_out`
 *   cache_out    NULL, or a cache that receives the pooled entries, the raw
 *                window, the open block's pooling state and seq_lens = T, so
 *                that lbca_append / lbca_decode continue the sequences
 *   workspace    device, lbca_prefill_workspace_bytes(cfg, B, T, cache_out != NULL)
 *   d_status     nullable device word for device-side conditions (a bounded
 *                wait of the tensor-core kernel giving up: LBCA_ERR_TIMEOUT; a
 *                query, key or value beyond the fp16 range of its tensor-core
 *                operands, |x| > 65504 after RoPE: LBCA_ERR_UNSUPPORTED, the
 *                output then not valid)
 * bf16 I/O with D = 128, no RMSNorm and separate K/V runs QK^T and PV on the
 * tensor cores (tcgen05, TMEM accumulators, TMA-fed tiles); every other
 * shape runs the f32 CUDA-core kernel (no TF32).
 * Errors: LBCA_ERR_ARG, LBCA_ERR_ALIGN, LBCA_ERR_CAPACITY (cache too small),
 * LBCA_ERR_UNSUPPORTED, LBCA_ERR_CUDA.
 */
LBCA_API lbca_status lbca_prefill(const lbca_config* cfg, const void* q, const void* k, const void* v,
                         const void* zk, const void* zv, const void* b_pos_k,
                         const void* b_pos_v, const float* sink, const void* gamma_q,
                         const void* gamma_kv, int32_t batch, int32_t T, void* out,
                         const lbca_cache* cache_out, void* workspace, size_t workspace_bytes,
                         int32_t* d_status, lbca_stream_t stream);

/*
 * lbca_prefill_rows -- the prefill's attention for a range of query rows, from
 * pooled entries and raw tokens the caller assembles: the building block of a
 * context-parallel prefill, where each rank owns a block-aligned range of
 * tokens, pools it (lbca_pool with pos0 = its first token), all-gathers the
 * pooled entries and receives the previous rank's last n_win + m - 1 raw
 * tokens (mSeek README, "How LBCA works", steps 4-5; same visible set and
 * arithmetic as lbca_prefill, on the CUDA cores).
 *   q, out     device [B, n_rows, Hq, D]: rows at absolute positions row0 ..
 *              row0 + n_rows - 1
 *   k, v       device [B, n_raw, G, D] raw keys and values at absolute
 *              positions raw0 .. raw0 + n_raw - 1, with raw0 + n_raw = row0 +
 *              n_rows and raw0 <= P(row0 + 1) m (the first row's window start;
 *              raw0 = max(0, row0 - (n_win + m - 1)) always qualifies);
 *              shared form: k = C, v = NULL
 *   pooled_k/v device [B, G, pool_stride, D] f32 finalised pooled entries of
 *              blocks 0 .. P(row0 + n_rows) - 1 (lbca_pool_f32); shared
 *              form: pooled_v = NULL
 * Errors: LBCA_ERR_ARG (a span that does not cover the rows' visible sets),
 * LBCA_ERR_ALIGN, LBCA_ERR_UNSUPPORTED, LBCA_ERR_CUDA.
 */
LBCA_API lbca_status lbca_prefill_rows(const lbca_config* cfg, const void* q, int32_t row0, int32_t n_rows,
                                       const void* k, const void* v, int32_t raw0, int32_t n_raw,
                                       const float* pooled_k, const float* pooled_v, int32_t pool_stride,
                                       const float* sink, const void* gamma_q, const void* gamma_kv, int32_t batch,
                                       void* out, lbca_stream_t stream);

/*
 * lbca_prefill_backward -- gradients of the prefill for training (mSeek
 * README, "Experiment at a glance": the LBCA layers are trained by continued
 * pretraining; the forward is lbca_prefill's).  Given dout [B, T, Hq, D], the
 * gradient of a loss with respect to every output row of lbca_prefill on the
 * same inputs, writes the gradients of that loss with respect to
 *   dq        [B, T, Hq, D]  the queries
 *   dk, dv    [B, T, G, D]   the raw keys and values (shared form: dk is the
 *                            gradient of C, dv NULL)
 *   dzk, dzv  [B, T, G, D]   the pooling logits (zero for tokens of the open
 *                            block, which is never pooled)
 *   db_pos_k/_v [m, G*D]     the positional biases
 *   dsink     [Hq]           the sink logits (NULL when sink is NULL)
 * all f32, device, overwritten (RMSNorm gains are not differentiated).  The
 * inputs are lbca_prefill's (I/O dtype); arithmetic is f32 on the CUDA cores:
 * the pooled entries, finalised keys and queries and the attention output are
 * recomputed in f32 in `workspace` (>= lbca_prefill_backward_workspace_bytes
 * bytes), then dq per query row, dkey and dvalue per entry over the contiguous
 * range of rows that see it, back through RoPE and RMSNorm, then through the
 * pooling softmax.  D in {32, 64, 128, 256, 512} (else LBCA_ERR_UNSUPPORTED).
 */
LBCA_API size_t lbca_prefill_backward_workspace_bytes(const lbca_config* cfg, int32_t batch, int32_t T);
LBCA_API lbca_status lbca_prefill_backward(const lbca_config* cfg, const void* q, const void* k, const void* v,
                                           const void* zk, const void* zv, const void* b_pos_k,
                                           const void* b_pos_v, const float* sink, const void* gamma_q,
                                           const void* gamma_kv, const void* dout, int32_t batch, int32_t T,
                                           float* dq, float* dk, float* dv, float* dzk, float* dzv,
                                           float* db_pos_k, float* db_pos_v, float* dsink, void* workspace,
                                           size_t workspace_bytes, lbca_stream_t stream);

/*
 * lbca_decode_noalloc -- lbca_decode for callers that cannot allocate.
 * The pages have no counterpart of this entry point; it exists for callers
 * that are not allowed to allocate device memory at all -- for example code
 * running inside a host framework that owns every device allocation, or a
 * serving loop that must not allocate once it is running -- and so have no
 * workspace to hand to lbca_decode.  It computes exactly what lbca_decode
 * computes, with the same arguments minus the workspace; the split partials
 * and merge counters live in a static device array of the library
 * (LBCA_NOALLOC_SCRATCH_BYTES, held by every GPU that loads the library until
 * the process exits).
 *   - A call whose split partials would need more than that returns
 *     LBCA_ERR_CAPACITY (use lbca_decode with a workspace instead).
 *   - The first call on a device looks up the array's device address; make
 *     that first call before any stream capture on that device.
 *   - No cudaMalloc, cudaFree or other allocating routine is called; each
 *     call zeroes the merge counters with an asynchronous memset on `stream`.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents: calls that overlap on the GPU (other streams, other host
 *     threads) race and corrupt each other's results.
 *   - The looked-up address, like the kernel attributes every entry point sets
 *     once per device, belongs to the device's current context: after a
 *     cudaDeviceReset the process must not call the library on that device
 *     again (the cached address and attributes are stale).
 */
#define LBCA_NOALLOC_SCRATCH_BYTES (8u << 20)
LBCA_API lbca_status lbca_decode_noalloc(const lbca_config* cfg, const void* q, const lbca_cache* cache,
                                         const float* sink, const void* gamma_q, const void* gamma_kv,
                                         int32_t max_ctx, void* out,
                                         int32_t* d_status, lbca_stream_t stream);

/*
 * lbca_selftest_bounded_wait -- check of the bounded device-side wait.
 * The pages have no counterpart; it exists so that the timeout path of the
 * kernels' waits can be exercised without a fault.  One CTA waits, with the
 * helper every kernel uses, on an mbarrier that nothing arrives at (arrive =
 * 0) or that its own thread completes first (arrive = 1, the control); after
 * limit_ns nanoseconds of wall time (1 .. 2e9) the wait gives up and
 * LBCA_ERR_TIMEOUT is written to the device word d_status (required).  The
 * kernel returns normally either way, so the context stays usable.
 */
LBCA_API lbca_status lbca_selftest_bounded_wait(int32_t arrive, uint64_t limit_ns, int32_t* d_status,
                                                lbca_stream_t stream);

/*
 * lbca_decode_sparse -- core attention of the CSA form for one query per
 * sequence over the selected compressed entries plus the raw window (CSA page,
 * "What is implemented", Eqs 18-19 and Eq 27: one key/value entry shared by
 * all heads, each selected compressed entry used as key and as value, a
 * window branch over the n_win most recent raw tokens, RMSNorm of queries and
 * entries, RoPE on the last dims with the outputs turned back by -t, and a
 * sink logit).
 *   q        device [B, Hq, D] queries at position t = seq_lens[b] - 1
 *   cache    pooled_k holds the finalised compressed entries (lbca_pool_dual,
 *            LBCA_KEY); ring_k the raw entries of (at least) the last n_win
 *            tokens, token s in slot s % ring_slots (ring_slots >= n_win)
 *   sel      device [B, top_k] int32: the selected block indices (as
 *            lbca_indexer_topk writes them: valid ones first); the first
 *            min(top_k, floor(L / m), max_blocks) are used
 *   out      device [B, Hq, D]
 * One softmax over the selected entries, the window tokens s in
 * [max(0, L - n_win), t] (finalised in f32 when read: RMSNorm, RoPE at s) and
 * the sink; a window token may also be summarised by a selected entry (the
 * two branches overlap).  The output's RoPE dims turn back by -t.  Runs on the
 * tensor-core shared-entry kernel: bf16, 64 query heads per kv head, D 256 or
 * 512, top_k + n_win within its cluster capacity (else LBCA_ERR_UNSUPPORTED).
 * A selected index outside [0, max_blocks) sets d_status to LBCA_ERR_ARG (its
 * row counts as zeros).
 */
LBCA_API lbca_status lbca_decode_sparse(const lbca_config* cfg, const void* q, const lbca_cache* cache,
                                        const int32_t* sel, int32_t top_k, const float* sink, const void* gamma_q,
                                        const void* gamma_kv, void* out, int32_t* d_status, lbca_stream_t stream);

/*
 * lbca_indexer_topk -- lightning-indexer relevance and top-k block selection
 * for one query per sequence (the CSA form; CSA page, "What is implemented",
 * Eqs 13-17: each indexer head scores a compressed indexer key by the ReLU of
 * its dot product with a low-rank indexer query, learned per-head weights
 * combine the heads, and the k best of the blocks the query may causally see
 * are kept).
 *   q_idx      device [B, n_heads, head_dim] bf16 indexer queries
 *   w_idx      device [B, n_heads] f32 head weights
 *   k_idx      device [B, max_blocks, head_dim] bf16 compressed indexer keys
 *              (e.g. lbca_pool_dual of the indexer key series, LBCA_VALUE)
 *   seq_lens   device [B] tokens the query sees (L); blocks j < floor(L /
 *              block_m), capped at max_blocks, are visible
 *   sel        device [B, top_k] int32 out: the selected block indices in
 *              increasing order (equal relevances: lower index first), then
 *              -1 where fewer than top_k blocks are visible
 *   sel_scores device [B, top_k] f32 out (nullable): their relevances
 *   workspace  device, >= lbca_indexer_workspace_bytes(B, max_blocks) bytes
 * Relevance of block j: I_j = sum_h w_h ReLU(q_h . k_j) (f32 accumulation of
 * exact bf16 products on the tensor cores).  Shapes: n_heads 32, 64 or 128;
 * head_dim 64 or 128 (else LBCA_ERR_UNSUPPORTED).
 */
LBCA_API size_t lbca_indexer_workspace_bytes(int32_t batch, int32_t max_blocks);
LBCA_API lbca_status lbca_indexer_topk(int32_t batch, int32_t n_heads, int32_t head_dim, int32_t block_m,
                                       int32_t top_k, const void* q_idx, const float* w_idx, const void* k_idx,
                                       int32_t max_blocks, const int32_t* seq_lens, int32_t* sel,
                                       float* sel_scores, void* workspace, size_t workspace_bytes,
                                       int32_t* d_status, lbca_stream_t stream);

/* Static text for a status code. */
LBCA_API const char* lbca_status_string(lbca_status status);

#ifdef __cplusplus
}
#endif

#endif /* LBCA_H */
