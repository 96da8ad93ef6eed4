/*
 * spla.h -- C ABI of the SPLA decode library (libspla.so), sm_100a (B200).
 *
 * The method is "SPLA: Block Sparse Plus Linear Attention for Long Context
 * Modeling" (gist.science technical summary, sections 2.1-2.3). One decode
 * step, for every query head:
 *   a1  score every KV block with the log of the second-order Taylor estimate
 *       n_j exp(q'.mu_j)(1 + 1/2 q'^T diag(sigma_j^2) q'), q' = q * softmax_scale
 *       (section 2.1);
 *   a2  keep the top_k blocks (plus sink/local blocks when asked for);
 *   a3  exact softmax attention over the kept blocks (section 2, opening);
 *   a4  residual linear attention over the blocks not kept, by subtraction:
 *       o_rla = (N - N~)/(D - D~), N, D from the global state S, z and
 *       N~, D~ from the kept blocks, feature map phi = exp (section 2.2);
 *   a5  out = o_sparse + gamma * RMSNorm(o_rla) (section 2.3).
 * The state a4 reads is kept current by spla_append_kv (a0).
 *
 * Conventions
 *   Memory.   Every pointer argument is DEVICE memory owned by the caller,
 *             unless a comment says "host". The library allocates nothing and
 *             never synchronises; all work is enqueued on `stream` (a
 *             cudaStream_t passed as void*; NULL = legacy default stream).
 *             spla_decode needs q and the cache's pools, statistics, S, z and
 *             m 16-byte aligned (it moves them with bulk copies and 16-byte
 *             loads); the append calls need the pools and S 16-byte aligned.
 *             Each returns SPLA_ERR_INVALID_ARG otherwise.
 *   Errors.   Argument errors are returned synchronously, before any CUDA
 *             call, and nothing is enqueued. Faults the kernels detect
 *             (a block-table entry out of range, a length past the table's
 *             capacity, a bounded wait that ran out) are OR-ed into
 *             *dev_status as SPLA_DEV_* bits; the caller reads it after its
 *             own synchronisation. Kernels never trap.
 *   Shapes.   Hq = num_q_heads, Hkv = num_kv_heads, G = Hq/Hkv (1, 2 or 4),
 *             d = head_dim (64 or 128), B = block_size (64 or 128).
 *   Dtypes.   q, K, V and out share params->dtype (SPLA_F32 or SPLA_BF16);
 *             block statistics and the linear-attention state are fp32.
 */
#ifndef SPLA_H
#define SPLA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPLA_API __attribute__((visibility("default")))
#else
#define SPLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SPLA_OK = 0,
    SPLA_ERR_INVALID_ARG = 1,   /* null pointer, bad size or inconsistent shape */
    SPLA_ERR_UNSUPPORTED = 2,   /* shape outside what the kernels implement */
    SPLA_ERR_WORKSPACE = 3,     /* workspace null or smaller than spla_decode_workspace_size */
    SPLA_ERR_CAPACITY = 4,      /* a host-known size exceeds a fixed limit */
    SPLA_ERR_CUDA = 5           /* a CUDA runtime call failed; see spla_last_cuda_error() */
} spla_status;

/* Bits the kernels OR into *dev_status. */
#define SPLA_DEV_BAD_BLOCK_TABLE 0x1   /* a block-table entry outside [0, num_phys_blocks) */
#define SPLA_DEV_CAPACITY        0x2   /* a length or an append past max_blocks_per_seq*B */
#define SPLA_DEV_TIMEOUT         0x4   /* a bounded wait on a TMA barrier ran out */
#define SPLA_DEV_BAD_COUNT       0x8   /* n_new[b] outside [0, max_new] */
#define SPLA_DEV_RLA_UNRESOLVED  0x10  /* a head's residual denominator D - D~ was not positive:
                                          its o_rla was set to 0 (see spla_decode) */

typedef enum { SPLA_F32 = 0, SPLA_BF16 = 1 } spla_dtype;

/* params->flags */
#define SPLA_FLAG_NO_RLA      0x1u  /* "SPA" ablation of section 4: o_rla = 0, out = o_sparse */
#define SPLA_FLAG_FIRST_ORDER 0x2u  /* mean-only score (first-order ablation of section 4) */

/* Largest max_blocks_per_seq the selection kernel handles. */
#define SPLA_MAX_BLOCKS_PER_SEQ 32768

typedef struct {
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim;        /* 64 or 128 */
    int32_t block_size;      /* 64 or 128 */
    int32_t top_k;           /* >= 1 */
    int32_t n_sink;          /* first n_sink blocks always kept (0 unless a workload asks) */
    int32_t n_local;         /* last n_local blocks always kept */
    int32_t dtype;           /* spla_dtype */
    float softmax_scale;     /* <= 0: 1/sqrt(head_dim) */
    float rms_eps;           /* <= 0: 1e-6 */
    uint32_t flags;          /* SPLA_FLAG_* */
} spla_params;

/*
 * The paged KV cache and its per-block statistics and global state. All
 * buffers are caller-allocated device memory; spla_cache_init prepares them.
 *   k_pool, v_pool : [num_phys_blocks][Hkv][B][d], params->dtype. Slots past a
 *                    sequence's length may hold anything.
 *   blk_stats      : [batch][Hkv][max_blocks_per_seq][2][d] fp32, indexed by
 *                    LOGICAL block: key mean, then key population variance, of
 *                    the block's stored tokens. Kept in logical order so that
 *                    one sequence's statistics stream contiguously whatever the
 *                    physical order of its KV blocks.
 *   S              : [batch][Hkv][d][d] fp32, sum_t exp(k_t - m) v_t^T
 *   z, m           : [batch][Hkv][d] fp32, sum_t exp(k_t - m) and the running
 *                    per-dimension max of k (the state's scaling).
 *   block_table    : [batch][max_blocks_per_seq] int32, logical -> physical block.
 *   context_lens   : [batch] int32 tokens held; advanced by spla_append_kv.
 */
typedef struct {
    void* k_pool;
    void* v_pool;
    float* blk_stats;
    float* S;
    float* z;
    float* m;
    const int32_t* block_table;
    int32_t* context_lens;
    int32_t batch;
    int32_t max_blocks_per_seq;
    int32_t num_phys_blocks;
} spla_cache;

/*
 * Empty every sequence: context_lens = 0, S = 0, z = 0, m = -inf.
 * Pools and statistics are left as they are (slots are rewritten on append).
 */
SPLA_API spla_status spla_cache_init(const spla_params* params, const spla_cache* cache, void* stream);

/*
 * a0 -- append tokens and keep the block statistics and the global state current
 * (section 2.1: mean and diagonal variance per block; section 2.2: the global
 * linear-attention state accumulates phi(k) v^T and phi(k) over every token).
 *   k_new, v_new : [batch][max_new][Hkv][d], params->dtype; sequence b uses
 *                  its first n_new[b] rows.
 *   n_new        : [batch] int32 (device), each in [0, max_new].
 *   max_new      : host int, >= 0; bounds the launch grid.
 *   dev_status   : int32 (device), OR-ed with SPLA_DEV_* bits; may be NULL.
 * For every sequence: tokens go to slots context_lens[b] .. + n_new[b] - 1
 * through block_table; the statistics of every block touched are recomputed
 * from all of its tokens; m rises to cover the new keys, S and z are rescaled
 * by exp(m_old - m_new) and the new tokens added; context_lens[b] advances.
 * A sequence whose append would pass max_blocks_per_seq*B, or whose n_new is
 * out of range, is left unchanged and flagged.
 */
SPLA_API spla_status spla_append_kv(const spla_params* params, const spla_cache* cache,
                           const void* k_new, const void* v_new, const int32_t* n_new,
                           int32_t max_new, int32_t* dev_status, void* stream);

/*
 * a0 for many tokens per call (a prefill, or a long chunk) -- the same result as
 * spla_append_kv up to fp32 rounding order, with the global state's sum over the
 * new tokens, phi(K)^T V, run as a dense contraction on the tensor cores (section
 * 2.2: the state accumulates phi(k) v^T over every token; section 2.3: phi = exp).
 * Arguments as for spla_append_kv, plus:
 *   workspace       : device scratch of at least spla_append_bulk_workspace_size
 *                     bytes, 16-byte aligned, owned by the caller; the call reads
 *                     and writes it on `stream` only, so calls on one stream may
 *                     share it. Its contents need no initialisation.
 * Supported: params->dtype == SPLA_BF16 and head_dim == 128 (SPLA_ERR_UNSUPPORTED
 * otherwise; spla_append_kv covers every shape); k_new and v_new 16-byte aligned
 * (SPLA_ERR_INVALID_ARG otherwise). The new tokens of a sequence are cut into
 * splits of whole 64-token tiles; every split's partial state (S_c, z_c at its
 * own maximum m_c) is merged into S, z, m in split order, so repeated calls give
 * bit-identical results. Device faults as for spla_append_kv.
 */
SPLA_API spla_status spla_append_kv_bulk(const spla_params* params, const spla_cache* cache,
                                const void* k_new, const void* v_new, const int32_t* n_new,
                                int32_t max_new, void* workspace, size_t workspace_bytes,
                                int32_t* dev_status, void* stream);

/*
 * Bytes of scratch spla_append_kv_bulk needs for (batch, max_new) under params
 * (host-only, no CUDA call; depends only on its arguments).
 */
SPLA_API spla_status spla_append_bulk_workspace_size(const spla_params* params, int32_t batch,
                                            int32_t max_new, size_t* bytes);

/*
 * Layout facts of the decode workspace that callers may rely on (measurement and
 * tests; the rest of the workspace is private):
 *   bytes [0, SPLA_WS_STAMP_BYTES): device timestamps of the last call's kernels
 *     (written only while spla_profile_stamps is on for the calling thread),
 *     uint64 [4 kernels: scoring, selection, decode, combine][256 SM slots][2]: per SM, ~t
 *     of the first CTA past its dependency wait and t of the last CTA's exit, ns of
 *     %globaltimer, raised with atomicMax (the kernel's span is the maximum of the
 *     first entries, complemented, to the maximum of the second). A caller that
 *     reads them zeroes these bytes before the call; nothing else depends on them.
 *   from byte SPLA_WS_STAMP_BYTES: the last call's block scores (log of the Taylor
 *     estimate), fp32 [batch][Hq][ld], ld = max_blocks_per_seq rounded up to a
 *     multiple of 4; entries past a sequence's blocks are undefined.
 */
#define SPLA_WS_STAMP_BYTES 16384u

/*
 * Bytes of scratch spla_decode needs for this shape (host-only, no CUDA call).
 * The value depends only on its arguments.
 */
SPLA_API spla_status spla_decode_workspace_size(const spla_params* params, int32_t batch,
                                       int32_t max_blocks_per_seq, size_t* bytes);

/*
 * a1..a5 -- one decode step for every (sequence, query head).
 *   q          : [batch][Hq][d], params->dtype.
 *   rms_gamma  : [Hq][d] fp32 RMSNorm scale, or NULL for ones.
 *   out        : [batch][Hq][d], params->dtype.
 *   sel_idx    : [batch][Hq][top_k + n_sink + n_local] int32 or NULL: the
 *                blocks kept, ascending, padded with -1.
 *   o_sparse_dbg, o_rla_dbg : [batch][Hq][d] fp32 or NULL: the two branches
 *                before the combine.
 *   workspace  : device scratch of >= spla_decode_workspace_size bytes,
 *                256-byte aligned; its contents need no initialisation. Calls
 *                that share a workspace must be ordered on the GPU (one stream,
 *                or events).
 *   dev_status : int32 (device) or NULL.
 * Decode attends over tokens [0, context_lens[b]). An empty sequence gives
 * out = 0. o_rla is 0 when every block is kept. When the residual denominator
 * D - D~ (the linear-attention mass of the blocks not kept, by subtraction) is
 * not positive in the arithmetic of the kernels, the unkept mass is below the
 * state's resolution: that head's o_rla is set to 0 and SPLA_DEV_RLA_UNRESOLVED
 * is OR-ed into *dev_status. Selection ties go to the lower block index.
 */
SPLA_API spla_status spla_decode(const spla_params* params, const spla_cache* cache, const void* q,
                        const float* rms_gamma, void* out, int32_t* sel_idx,
                        float* o_sparse_dbg, float* o_rla_dbg,
                        void* workspace, size_t workspace_bytes,
                        int32_t* dev_status, void* stream);

/*
 * Context-sharded decode (one long sequence over several GPUs, or several caches):
 * the method's decode step split into three phases with an exchange between
 * them. Shard s holds the global blocks [first_block, first_block +
 * max_blocks_per_seq) of every sequence in a cache of its own (pools,
 * statistics, and S, z, m over its own tokens; context_lens = its tokens);
 * global_nb [batch] (device int32) is each sequence's total block count. The
 * sink and local blocks are those of the whole sequence. Every shard passes the
 * same params, batch and query q. The kept set equals the unsharded one: the
 * sequence's top_k is the top_k of the union of the shards' local top_k. This
 * is the library's own split of the step over devices (the pages describe the
 * single-device step: section 2.1 selection, section 2.2 the residual by
 * subtraction, section 2.3 the output).
 *
 * 1. spla_shard_candidates: scores this shard's blocks and writes, per
 *    (sequence, query head), its best top_k blocks that are not sink or local
 *    blocks, best first (score descending, ties to the lower global block),
 *    padded with block = -1: cand [batch][Hq][top_k].
 * 2. The caller gathers every shard's cand into cand_all [nshards][batch][Hq][top_k]
 *    (an all-gather); nshards * top_k <= 4096.
 * 3. spla_shard_partials: with the same workspace as step 1, untouched in
 *    between, keeps this shard's forced blocks and those at or above the
 *    sequence's top_k-th candidate, decodes them and writes one record per
 *    (sequence, query head): part [batch][Hq][SPLA_SHARD_REC(d)] fp64.
 * 4. The caller gathers every shard's part into part_all [nshards][batch][Hq][...].
 * 5. spla_shard_merge: out (and the debug outputs) as spla_decode defines them
 *    (the same values up to the order of the fp32 sums), from part_all; any
 *    stream, no cache needed.
 * The workspace is spla_decode_workspace_size(params, batch, max_blocks_per_seq)
 * bytes. Argument checks and device faults as for spla_decode;
 * SPLA_ERR_CAPACITY when nshards * top_k exceeds 4096.
 */
typedef struct {
    float score;      /* the block's score (log of the Taylor estimate) */
    int32_t block;    /* global block index, -1 for none */
} spla_candidate;

#define SPLA_SHARD_REC(d) (8 + 2 * (d))

SPLA_API spla_status spla_shard_candidates(const spla_params* params, const spla_cache* cache,
                                  int32_t first_block, const int32_t* global_nb,
                                  const void* q, spla_candidate* cand, void* workspace,
                                  size_t workspace_bytes, int32_t* dev_status, void* stream);

SPLA_API spla_status spla_shard_partials(const spla_params* params, const spla_cache* cache,
                                int32_t first_block, const int32_t* global_nb, const void* q,
                                const spla_candidate* cand_all, int32_t nshards, double* part,
                                void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                void* stream);

SPLA_API spla_status spla_shard_merge(const spla_params* params, int32_t batch,
                             const double* part_all, int32_t nshards, const float* rms_gamma,
                             void* out, float* o_sparse_dbg, float* o_rla_dbg,
                             int32_t* dev_status, void* stream);

/*
 * The block-causal form over whole sequences (a prefill or training forward):
 * query t of sequence b sees its tokens 0..t. Its own block J = t / B is
 * attended exactly and causally; the complete earlier blocks 0..J-1 are scored
 * (section 2.1) and the sink blocks plus the top_k of the rest attended exactly
 * (ties to the lower block); the earlier blocks left out are covered by linear
 * attention by subtraction (section 2.2) from the state of the tokens before
 * block J; out = o_sparse + gamma * RMSNorm(o_rla) (section 2.3).
 *   cache       : holds exactly each sequence's tokens 0..context_lens[b]-1,
 *                 appended from k_all / v_all (its statistics, pools and final m
 *                 are used; n_local is ignored: the query's own block plays it).
 *   k_all, v_all: [batch][max_len][Hkv][d] bf16, the same tokens; q_all
 *                 [batch][max_len][Hq][d] bf16; all 16-byte aligned.
 *   out         : [batch][max_len][Hq][d] bf16; rows t >= context_lens[b] are not
 *                 written. o_sparse_dbg, o_rla_dbg: the same layout in fp32, or NULL.
 *   workspace   : spla_block_causal_workspace_size bytes, 256-byte aligned: per
 *                 block states and the prefix states at every block boundary.
 * Supported: bf16, head_dim 128, at most 4096 blocks per sequence, top_k <= 256
 * (SPLA_ERR_UNSUPPORTED / SPLA_ERR_CAPACITY otherwise). Device faults as for
 * spla_decode (a residual the fp32 sums cannot resolve sets
 * SPLA_DEV_RLA_UNRESOLVED and gives o_rla = 0 for that query and head).
 */
SPLA_API spla_status spla_block_causal_workspace_size(const spla_params* params, int32_t batch,
                                             int32_t max_len, size_t* bytes);

SPLA_API spla_status spla_block_causal_forward(const spla_params* params, const spla_cache* cache,
                                      const void* k_all, const void* v_all, const void* q_all,
                                      int32_t max_len, const float* rms_gamma, void* out,
                                      float* o_sparse_dbg, float* o_rla_dbg, void* workspace,
                                      size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * Bytes of the library-owned scratch that spla_decode_static_workspace uses
 * on each device (one file-scope __device__ array, 256-byte aligned).
 */
#define SPLA_STATIC_WORKSPACE_BYTES (16u << 20)

/*
 * spla_decode without a caller workspace: the method has no counterpart (the
 * pages do not speak of memory management); this is a convenience of the
 * library. It serves callers that cannot allocate device memory where they
 * decode: a plain C host program with no device allocator of its own, or a
 * serving engine whose KV-cache pool took all free HBM at start-up. It
 * allocates nothing; the scratch is a SPLA_STATIC_WORKSPACE_BYTES array built
 * into the library, one per device.
 *   Arguments, results and dev_status are those of spla_decode; the work is
 *   enqueued on `stream`, which must belong to the current device.
 *   Size limit: a shape whose spla_decode_workspace_size exceeds
 *   SPLA_STATIC_WORKSPACE_BYTES returns SPLA_ERR_CAPACITY on the host, before
 *   any CUDA call, and enqueues nothing.
 *   First call per device: it looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current, and keeps it together
 *   with the id of the device's context; a call that finds another context
 *   current (after cudaDeviceReset, say, which reloads the module) looks it
 *   up again. Make the first call in each context before any stream capture
 *   on the device. A failed lookup returns SPLA_ERR_CUDA.
 *   Sharing: every call on a device uses the same array. Nothing in it needs
 *   to start at zero (each kernel writes its scratch before the next one reads
 *   it), so it is never cleared. Calls whose kernels overlap on the GPU (on
 *   streams with no ordering between them) race on it.
 */
SPLA_API spla_status spla_decode_static_workspace(const spla_params* params,
                                         const spla_cache* cache, const void* q,
                                         const float* rms_gamma, void* out, int32_t* sel_idx,
                                         float* o_sparse_dbg, float* o_rla_dbg,
                                         int32_t* dev_status, void* stream);

/*
 * Measurement hook (no part of the method). With 2 <= n <= 8, every later
 * spla_decode call made from this host thread records events[0..n-1]
 * (cudaEvent_t handles) on its stream: events[0] before its first kernel and
 * events[i] after its i-th kernel; events past the call's last kernel are
 * recorded right after it. spla_decode runs four kernels: scoring, selection,
 * split-KV decode and combine. n == 0 turns it off. The handles are copied; the events stay the caller's. Returns
 * SPLA_ERR_INVALID_ARG for any other n or a NULL array or handle.
 */
SPLA_API spla_status spla_profile_events(void* const* events, int32_t n);

/*
 * Measurement hook (no part of the method). With on != 0, later spla_decode calls
 * made from this host thread write their kernels' device timestamps into the
 * first SPLA_WS_STAMP_BYTES of the workspace (see SPLA_WS_STAMP_BYTES); with
 * on == 0 (the default) the kernels skip them.
 */
SPLA_API spla_status spla_profile_stamps(int32_t on);

/* Human-readable name of a status (static storage). */
SPLA_API const char* spla_status_string(spla_status s);

/* The cudaError_t of the last CUDA call that failed in this thread (0 if none). */
SPLA_API int32_t spla_last_cuda_error(void);

/* Library version, major*10000 + minor*100 + patch. */
SPLA_API int32_t spla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPLA_H */
