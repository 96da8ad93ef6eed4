// Host side of the C ABI declared in include/spla.h: argument checks,
// workspace layout, TMA descriptors and the launch sequence.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <mutex>

#include "common.cuh"

namespace spla {
cudaError_t launch_cache_init(const CacheView& c, cudaStream_t s);
cudaError_t launch_append(const CacheView& c, int dtype, const void* k_new, const void* v_new,
                          const int32_t* n_new, int32_t max_new, int32_t* status, cudaStream_t s);
cudaError_t launch_append_bulk(const CacheView& c, const CUtensorMap& tk, const CUtensorMap& tv,
                               const void* k_new, const void* v_new, const int32_t* n_new,
                               int32_t max_new, float* part, int32_t* status, cudaStream_t s);
size_t bulk_workspace_bytes(int batch, int hkv, int d, int max_new);
int shard_max_gathered();
int bc_max_blocks();
int bc_max_top_k();
size_t bc_workspace_bytes(int batch, int hkv, int bs, int max_len);
cudaError_t launch_block_causal_entry(const CacheView& c, const CUtensorMap& tk,
                                      const CUtensorMap& tv, const void* k_all, int32_t max_len,
                                      const void* q_all, const float* gamma, void* out,
                                      float* o_sp, float* o_rl, int top_k, int n_sink,
                                      int first_order, int no_rla, double scale, float eps,
                                      char* ws, int32_t* status, cudaStream_t s);
cudaError_t launch_shard_cand(const CacheView& c, const float* scores, int ld,
                              const uint32_t* bits, int nw, int top_k, int n_sink, int n_local,
                              int32_t first_block, const int32_t* global_nb, void* cand,
                              int32_t* status, cudaStream_t s);
cudaError_t launch_shard_mark(const CacheView& c, const float* scores, int ld,
                              const void* cand_all, int nshards, int top_k, int n_sink,
                              int n_local, int32_t first_block, const int32_t* global_nb,
                              uint32_t* bits, int nw, int32_t* nsel, cudaStream_t s);
cudaError_t launch_shard_partial(const CacheView& c, int dtype, const DecodeArgs& a,
                                 const void* q, double* rec, cudaStream_t s);
cudaError_t launch_shard_merge(int heads, int hq, int d, int dtype, const double* rec_all,
                               int nshards, int no_rla, float eps, const float* gamma, void* out,
                               float* o_sp, float* o_rl, int32_t* status, cudaStream_t s);
cudaError_t launch_score(const CacheView& c, const CUtensorMap& tstats, int dtype, const void* q,
                         double scale, int first_order, float* scores, int ld, float* gread,
                         float* aw, KernelStamps* stamps, int32_t* status, cudaStream_t s);
int score_readout_parts(int d);
cudaError_t launch_select(const CacheView& c, int top_k, int n_sink, int n_local,
                          const float* scores, int ld, uint32_t* bits, int nw, int32_t* nsel,
                          int32_t* sel_idx, int kcap, KernelStamps* stamps, cudaStream_t s);
cudaError_t launch_decode_mma(const CacheView& c, const CUtensorMap& tk, const CUtensorMap& tv,
                              const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_decode_simt(const CacheView& c, int dtype, const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_combine(const CacheView& c, int dtype, const DecodeArgs& a, cudaStream_t s);
size_t mma_smem_for(int d, int bs, int max_per);
size_t simt_smem_for(int d, int bs, int max_per);

// The split heuristic is tuned for the 148-SM B200 (three decode CTAs per SM);
// results do not depend on it.
constexpr int kTargetCtas = 148;
constexpr int kDecodeSlots = 3 * kTargetCtas;
constexpr int kMaxSplit = 512;
constexpr int kMaxSmem = 227 * 1024;

static thread_local int32_t g_last_cuda_error = 0;
constexpr int kMaxProfEvents = 8;
static thread_local cudaEvent_t g_prof[kMaxProfEvents] = {};
static thread_local int g_prof_n = 0;
static thread_local bool g_stamps_on = false;

// Event i (0 < i < n) is recorded after the i-th kernel of a decode call, event 0
// before the first; prof_done() records the ones a shorter chain did not reach.
static void prof_mark(int i, cudaStream_t s) {
    if (i < g_prof_n) cudaEventRecord(g_prof[i], s);
}
static void prof_done(int next, cudaStream_t s) {
    for (int i = next; i < g_prof_n; ++i) cudaEventRecord(g_prof[i], s);
}

void set_last_cuda_error(int32_t e) { g_last_cuda_error = e; }

static spla_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = (int32_t)e;
    return SPLA_ERR_CUDA;
}

static spla_status check_params(const spla_params* p) {
    if (!p) return SPLA_ERR_INVALID_ARG;
    if (p->num_q_heads <= 0 || p->num_kv_heads <= 0 || p->num_q_heads % p->num_kv_heads)
        return SPLA_ERR_INVALID_ARG;
    const int G = p->num_q_heads / p->num_kv_heads;
    if (G != 1 && G != 2 && G != 4) return SPLA_ERR_UNSUPPORTED;
    if (p->head_dim != 64 && p->head_dim != 128) return SPLA_ERR_UNSUPPORTED;
    if (p->block_size != 64 && p->block_size != 128) return SPLA_ERR_UNSUPPORTED;
    if (p->top_k < 1 || p->n_sink < 0 || p->n_local < 0) return SPLA_ERR_INVALID_ARG;
    if (p->dtype != SPLA_F32 && p->dtype != SPLA_BF16) return SPLA_ERR_UNSUPPORTED;
    if (p->flags & ~(SPLA_FLAG_NO_RLA | SPLA_FLAG_FIRST_ORDER)) return SPLA_ERR_INVALID_ARG;
    return SPLA_OK;
}

static spla_status check_cache(const spla_cache* c) {
    if (!c) return SPLA_ERR_INVALID_ARG;
    if (!c->k_pool || !c->v_pool || !c->blk_stats || !c->S || !c->z || !c->m ||
        !c->block_table || !c->context_lens)
        return SPLA_ERR_INVALID_ARG;
    if (c->batch <= 0 || c->max_blocks_per_seq <= 0 || c->num_phys_blocks <= 0)
        return SPLA_ERR_INVALID_ARG;
    if (c->max_blocks_per_seq > SPLA_MAX_BLOCKS_PER_SEQ) return SPLA_ERR_CAPACITY;
    return SPLA_OK;
}

// The append kernels read the pools back with 16-byte loads; the bulk merge moves
// S rows as 16-byte vectors.
static bool cache_aligned(const spla_cache* c) {
    auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) != 0; };
    return !(misaligned(c->k_pool) || misaligned(c->v_pool) || misaligned(c->S));
}

static CacheView view_of(const spla_params* p, const spla_cache* c) {
    CacheView v;
    v.k_pool = c->k_pool;
    v.v_pool = c->v_pool;
    v.stats = c->blk_stats;
    v.S = c->S;
    v.z = c->z;
    v.m = c->m;
    v.table = c->block_table;
    v.lens = c->context_lens;
    v.batch = c->batch;
    v.mbp = c->max_blocks_per_seq;
    v.num_phys = c->num_phys_blocks;
    v.hq = p->num_q_heads;
    v.hkv = p->num_kv_heads;
    v.group = p->num_q_heads / p->num_kv_heads;
    v.d = p->head_dim;
    v.bs = p->block_size;
    return v;
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static_assert((size_t)kStampCount * kStampSlots * sizeof(KernelStamps) <= SPLA_WS_STAMP_BYTES,
              "timestamp slots fit their region");

static DecodeLayout layout_of(const spla_params* p, int32_t batch, int32_t mbp) {
    DecodeLayout L;
    const int G = p->num_q_heads / p->num_kv_heads;
    const int groups = batch * p->num_kv_heads;
    L.kcap = p->top_k + p->n_sink + p->n_local;
    // a head's bitset row starts on 16 bytes (the decode kernel loads it as int4)
    L.nw = ((mbp + 31) / 32 + 3) & ~3;
    L.rec = rec_floats(p->head_dim);
    L.ld = (mbp + 3) & ~3;
    const int umax = (int)std::min<int64_t>(mbp, (int64_t)G * L.kcap);
    // one wave: as many splits per group as fit the resident CTA slots, at least 2 blocks each
    int ns = kDecodeSlots / groups;
    ns = std::max(1, std::min(ns, std::min(kMaxSplit, std::max(1, umax / 2))));
    L.nsplit = ns;
    L.max_per = (umax + ns - 1) / ns + 1;
    L.readout_parts = score_readout_parts(p->head_dim);
    // the first SPLA_WS_STAMP_BYTES receive the kernels' device timestamps
    size_t off = SPLA_WS_STAMP_BYTES;
    L.off_scores = off;
    off = align256(off + (size_t)batch * p->num_q_heads * L.ld * sizeof(float));
    L.off_bits = off;
    off = align256(off + (size_t)batch * p->num_q_heads * L.nw * sizeof(uint32_t));
    L.off_nsel = off;
    off = align256(off + (size_t)batch * p->num_q_heads * sizeof(int32_t));
    L.off_part = off;
    off = align256(off + (size_t)groups * ns * G * L.rec * sizeof(float));
    L.off_gread = off;
    off = align256(off + (size_t)groups * L.readout_parts * G * (p->head_dim + 4) * sizeof(float));
    L.off_aw = off;
    off = align256(off + (size_t)groups * p->head_dim * 4 * sizeof(float));
    L.total = off;
    return L;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 2-D view of a pool as [num_phys*Hkv*B rows][d cols] bf16; box = 64 rows x 64 cols (one
// 64-token pipeline unit of the decode kernel, 8 KiB), 128B swizzle.
static bool make_pool_map(CUtensorMap* m, const void* pool, const CacheView& c) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t rows = (cuuint64_t)c.num_phys * c.hkv * c.bs;
    cuuint64_t dims[2] = {(cuuint64_t)c.d, rows};
    cuuint64_t strides[1] = {(cuuint64_t)c.d * 2};
    cuuint32_t box[2] = {64u, 64u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(pool), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D view of the block statistics as [batch*Hkv*mbp rows][2d fp32 cols]; box = 32 rows x 32
// cols (the mean or the variance of 32 dimensions of 32 blocks, 4 KiB), 128B swizzle.
static bool make_stats_map(CUtensorMap* m, const CacheView& c) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(2 * c.d), (cuuint64_t)c.batch * c.hkv * c.mbp};
    cuuint64_t strides[1] = {(cuuint64_t)(2 * c.d) * 4};
    cuuint32_t box[2] = {32u, 32u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, c.stats, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D view of an append input [batch*max_new rows][Hkv][d] bf16; box = 64 dims x 1 head
// x 64 tokens (8 KiB), 128B swizzle; rows past the end read as zero.
static bool make_input_map(CUtensorMap* m, const void* x, const CacheView& c, int32_t max_new) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)c.d, (cuuint64_t)c.hkv, (cuuint64_t)c.batch * max_new};
    cuuint64_t strides[2] = {(cuuint64_t)c.d * 2, (cuuint64_t)c.hkv * c.d * 2};
    cuuint32_t box[3] = {64u, 1u, 64u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace spla

using namespace spla;

extern "C" {

int32_t spla_version(void) { return 100; }

const char* spla_status_string(spla_status s) {
    switch (s) {
        case SPLA_OK: return "ok";
        case SPLA_ERR_INVALID_ARG: return "invalid argument";
        case SPLA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case SPLA_ERR_WORKSPACE: return "workspace missing or too small";
        case SPLA_ERR_CAPACITY: return "size beyond a fixed limit";
        case SPLA_ERR_CUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

int32_t spla_last_cuda_error(void) { return g_last_cuda_error; }

spla_status spla_profile_events(void* const* events, int32_t n) {
    if (n == 0) {
        g_prof_n = 0;
        return SPLA_OK;
    }
    if (n < 2 || n > kMaxProfEvents || !events) return SPLA_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (!events[i]) return SPLA_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) g_prof[i] = (cudaEvent_t)events[i];
    g_prof_n = n;
    return SPLA_OK;
}

spla_status spla_profile_stamps(int32_t on) {
    g_stamps_on = on != 0;
    return SPLA_OK;
}

spla_status spla_cache_init(const spla_params* params, const spla_cache* cache, void* stream) {
    spla_status st = check_params(params);
    if (st != SPLA_OK) return st;
    if ((st = check_cache(cache)) != SPLA_OK) return st;
    const CacheView v = view_of(params, cache);
    cudaError_t e = launch_cache_init(v, (cudaStream_t)stream);
    return e == cudaSuccess ? SPLA_OK : cuda_fail(e);
}

spla_status spla_append_kv(const spla_params* params, const spla_cache* cache, const void* k_new,
                           const void* v_new, const int32_t* n_new, int32_t max_new,
                           int32_t* dev_status, void* stream) {
    spla_status st = check_params(params);
    if (st != SPLA_OK) return st;
    if ((st = check_cache(cache)) != SPLA_OK) return st;
    if (max_new < 0 || !n_new) return SPLA_ERR_INVALID_ARG;
    if (max_new > 0 && (!k_new || !v_new)) return SPLA_ERR_INVALID_ARG;
    if (!cache_aligned(cache)) return SPLA_ERR_INVALID_ARG;
    const CacheView v = view_of(params, cache);
    cudaError_t e = launch_append(v, params->dtype, k_new, v_new, n_new, max_new, dev_status,
                                  (cudaStream_t)stream);
    return e == cudaSuccess ? SPLA_OK : cuda_fail(e);
}

static spla_status check_bulk(const spla_params* params, int32_t batch, int32_t max_new) {
    spla_status st = check_params(params);
    if (st != SPLA_OK) return st;
    if (params->dtype != SPLA_BF16 || params->head_dim != 128) return SPLA_ERR_UNSUPPORTED;
    if (batch <= 0 || max_new < 0) return SPLA_ERR_INVALID_ARG;
    if ((int64_t)batch * max_new > INT32_MAX) return SPLA_ERR_CAPACITY;
    return SPLA_OK;
}

spla_status spla_append_bulk_workspace_size(const spla_params* params, int32_t batch,
                                            int32_t max_new, size_t* bytes) {
    spla_status st = check_bulk(params, batch, max_new);
    if (st != SPLA_OK) return st;
    if (!bytes) return SPLA_ERR_INVALID_ARG;
    *bytes = max_new > 0 ? bulk_workspace_bytes(batch, params->num_kv_heads, params->head_dim,
                                                max_new)
                         : 0;
    return SPLA_OK;
}

spla_status spla_append_kv_bulk(const spla_params* params, const spla_cache* cache,
                                const void* k_new, const void* v_new, const int32_t* n_new,
                                int32_t max_new, void* workspace, size_t workspace_bytes,
                                int32_t* dev_status, void* stream) {
    spla_status st = check_params(params);
    if (st != SPLA_OK) return st;
    if ((st = check_cache(cache)) != SPLA_OK) return st;
    if ((st = check_bulk(params, cache->batch, max_new)) != SPLA_OK) return st;
    if (!n_new || !cache_aligned(cache)) return SPLA_ERR_INVALID_ARG;
    const CacheView v = view_of(params, cache);
    cudaStream_t s = (cudaStream_t)stream;
    if (max_new == 0) {
        cudaError_t e = launch_append(v, params->dtype, k_new, v_new, n_new, 0, dev_status, s);
        return e == cudaSuccess ? SPLA_OK : cuda_fail(e);
    }
    if (!k_new || !v_new || (reinterpret_cast<uintptr_t>(k_new) & 15) ||
        (reinterpret_cast<uintptr_t>(v_new) & 15))
        return SPLA_ERR_INVALID_ARG;
    const size_t need = bulk_workspace_bytes(cache->batch, params->num_kv_heads, params->head_dim,
                                             max_new);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15))
        return SPLA_ERR_WORKSPACE;
    CUtensorMap tk, tv;
    if (!make_input_map(&tk, k_new, v, max_new) || !make_input_map(&tv, v_new, v, max_new))
        return SPLA_ERR_UNSUPPORTED;
    cudaError_t e = launch_append_bulk(v, tk, tv, k_new, v_new, n_new, max_new,
                                       reinterpret_cast<float*>(workspace), dev_status, s);
    return e == cudaSuccess ? SPLA_OK : cuda_fail(e);
}

spla_status spla_decode_workspace_size(const spla_params* params, int32_t batch,
                                       int32_t max_blocks_per_seq, size_t* bytes) {
    spla_status st = check_params(params);
    if (st != SPLA_OK) return st;
    if (!bytes || batch <= 0 || max_blocks_per_seq <= 0) return SPLA_ERR_INVALID_ARG;
    if (max_blocks_per_seq > SPLA_MAX_BLOCKS_PER_SEQ) return SPLA_ERR_CAPACITY;
    *bytes = layout_of(params, batch, max_blocks_per_seq).total;
    return SPLA_OK;
}

spla_status spla_decode(const spla_params* params, const spla_cache* cache, const void* q,
                        const float* rms_gamma, void* out, int32_t* sel_idx, float* o_sparse_dbg,
                        float* o_rla_dbg, void* workspace, size_t workspace_bytes,
                        int32_t* dev_status, void* stream) {
    spla_status st = check_params(params);
    if (st != SPLA_OK) return st;
    if ((st = check_cache(cache)) != SPLA_OK) return st;
    if (!q || !out) return SPLA_ERR_INVALID_ARG;
    // the kernels move these by bulk copies, TMA boxes and 16-byte vector loads
    auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) != 0; };
    if (misaligned(q) || misaligned(cache->S) || misaligned(cache->z) || misaligned(cache->m) ||
        misaligned(cache->blk_stats) || misaligned(cache->k_pool) || misaligned(cache->v_pool))
        return SPLA_ERR_INVALID_ARG;
    const DecodeLayout L = layout_of(params, cache->batch, cache->max_blocks_per_seq);
    if (!workspace || workspace_bytes < L.total) return SPLA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return SPLA_ERR_WORKSPACE;
    const CacheView v = view_of(params, cache);

    cudaStream_t s = (cudaStream_t)stream;
    char* ws = static_cast<char*>(workspace);
    float* scores = reinterpret_cast<float*>(ws + L.off_scores);
    uint32_t* bits = reinterpret_cast<uint32_t*>(ws + L.off_bits);
    int32_t* nsel = reinterpret_cast<int32_t*>(ws + L.off_nsel);
    float* part = reinterpret_cast<float*>(ws + L.off_part);
    const double scale = params->softmax_scale > 0.f ? (double)params->softmax_scale
                                                     : 1.0 / sqrt((double)params->head_dim);
    const float sl2 = (float)(scale * 1.4426950408889634);
    const float eps = params->rms_eps > 0.f ? params->rms_eps : 1e-6f;
    const int first_order = (params->flags & SPLA_FLAG_FIRST_ORDER) ? 1 : 0;
    const int no_rla = (params->flags & SPLA_FLAG_NO_RLA) ? 1 : 0;
    CUtensorMap tstats;
    if (!make_stats_map(&tstats, v)) return cuda_fail(cudaErrorInvalidValue);

    // ---- kernel chain: scoring, selection, split-KV decode, combine
    KernelStamps* stamps = g_stamps_on ? reinterpret_cast<KernelStamps*>(ws) : nullptr;
    const bool use_mma = params->dtype == SPLA_BF16;
    const size_t smem = use_mma ? mma_smem_for(v.d, v.bs, L.max_per)
                                : simt_smem_for(v.d, v.bs, L.max_per);
    if (smem > (size_t)kMaxSmem) return SPLA_ERR_CAPACITY;
    prof_mark(0, s);
    float* gread = reinterpret_cast<float*>(ws + L.off_gread);
    float* aw_ws = reinterpret_cast<float*>(ws + L.off_aw);
    cudaError_t e = launch_score(v, tstats, params->dtype, q, scale, first_order, scores, L.ld, gread,
                                 aw_ws, stamps, dev_status, s);
    if (e != cudaSuccess) return cuda_fail(e);
    prof_mark(1, s);
    e = launch_select(v, params->top_k, params->n_sink, params->n_local, scores, L.ld, bits, L.nw,
                      nsel, sel_idx, L.kcap, stamps, s);
    if (e != cudaSuccess) return cuda_fail(e);
    prof_mark(2, s);
    DecodeArgs da;
    da.q = q;
    da.gamma = rms_gamma;
    da.out = out;
    da.o_sp = o_sparse_dbg;
    da.o_rl = o_rla_dbg;
    da.bits = bits;
    da.nsel = nsel;
    da.part = part;
    da.gread = gread;
    da.status = dev_status;
    da.nw = L.nw;
    da.nsplit = L.nsplit;
    da.max_per = L.max_per;
    da.no_rla = no_rla;
    da.nrd = L.readout_parts;
    da.aw = aw_ws;
    da.stamps = stamps;
    da.sl2 = sl2;
    da.eps = eps;
    if (use_mma) {
        CUtensorMap tk, tv;
        if (!make_pool_map(&tk, v.k_pool, v) || !make_pool_map(&tv, v.v_pool, v))
            return cuda_fail(cudaErrorInvalidValue);
        e = launch_decode_mma(v, tk, tv, da, s);
    } else {
        e = launch_decode_simt(v, params->dtype, da, s);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    prof_mark(3, s);
    e = launch_combine(v, params->dtype, da, s);
    if (e != cudaSuccess) return cuda_fail(e);
    prof_mark(4, s);
    prof_done(5, s);
    return SPLA_OK;
}


// ------------------------------------------------------------------ context-sharded decode
// Checks shared by the two per-shard phases; fills the view, layout, scale.
static spla_status shard_setup(const spla_params* params, const spla_cache* cache, const void* q,
                               const int32_t* global_nb, int32_t first_block, void* workspace,
                               size_t workspace_bytes, CacheView* v, DecodeLayout* L) {
    spla_status st = check_params(params);
    if (st != SPLA_OK) return st;
    if ((st = check_cache(cache)) != SPLA_OK) return st;
    if (!q || !global_nb || first_block < 0) return SPLA_ERR_INVALID_ARG;
    auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) != 0; };
    if (misaligned(q) || misaligned(cache->S) || misaligned(cache->z) || misaligned(cache->m) ||
        misaligned(cache->blk_stats) || misaligned(cache->k_pool) || misaligned(cache->v_pool))
        return SPLA_ERR_INVALID_ARG;
    *L = layout_of(params, cache->batch, cache->max_blocks_per_seq);
    if (!workspace || workspace_bytes < L->total) return SPLA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return SPLA_ERR_WORKSPACE;
    *v = view_of(params, cache);
    return SPLA_OK;
}

spla_status spla_shard_candidates(const spla_params* params, const spla_cache* cache,
                                  int32_t first_block, const int32_t* global_nb, const void* q,
                                  spla_candidate* cand, void* workspace, size_t workspace_bytes,
                                  int32_t* dev_status, void* stream) {
    CacheView v;
    DecodeLayout L;
    spla_status st = shard_setup(params, cache, q, global_nb, first_block, workspace,
                                 workspace_bytes, &v, &L);
    if (st != SPLA_OK) return st;
    if (!cand) return SPLA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    char* ws = static_cast<char*>(workspace);
    float* scores = reinterpret_cast<float*>(ws + L.off_scores);
    uint32_t* bits = reinterpret_cast<uint32_t*>(ws + L.off_bits);
    int32_t* nsel = reinterpret_cast<int32_t*>(ws + L.off_nsel);
    float* gread = reinterpret_cast<float*>(ws + L.off_gread);
    float* aw_ws = reinterpret_cast<float*>(ws + L.off_aw);
    const double scale = params->softmax_scale > 0.f ? (double)params->softmax_scale
                                                     : 1.0 / sqrt((double)params->head_dim);
    const int first_order = (params->flags & SPLA_FLAG_FIRST_ORDER) ? 1 : 0;
    CUtensorMap tstats;
    if (!make_stats_map(&tstats, v)) return cuda_fail(cudaErrorInvalidValue);
    cudaError_t e = launch_score(v, tstats, params->dtype, q, scale, first_order, scores, L.ld,
                                 gread, aw_ws, nullptr, dev_status, s);
    if (e != cudaSuccess) return cuda_fail(e);
    // the shard's best top_k + n_sink + n_local blocks, nothing forced: they hold its
    // share of the sequence's top_k whatever the sink and local blocks are
    e = launch_select(v, L.kcap, 0, 0, scores, L.ld, bits, L.nw, nsel, nullptr, L.kcap, nullptr, s);
    if (e != cudaSuccess) return cuda_fail(e);
    e = launch_shard_cand(v, scores, L.ld, bits, L.nw, params->top_k, params->n_sink,
                          params->n_local, first_block, global_nb, cand, dev_status, s);
    return e == cudaSuccess ? SPLA_OK : cuda_fail(e);
}

spla_status spla_shard_partials(const spla_params* params, const spla_cache* cache,
                                int32_t first_block, const int32_t* global_nb, const void* q,
                                const spla_candidate* cand_all, int32_t nshards, double* part,
                                void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                void* stream) {
    CacheView v;
    DecodeLayout L;
    spla_status st = shard_setup(params, cache, q, global_nb, first_block, workspace,
                                 workspace_bytes, &v, &L);
    if (st != SPLA_OK) return st;
    if (!cand_all || !part || nshards < 1) return SPLA_ERR_INVALID_ARG;
    if ((int64_t)nshards * params->top_k > shard_max_gathered()) return SPLA_ERR_CAPACITY;
    cudaStream_t s = (cudaStream_t)stream;
    char* ws = static_cast<char*>(workspace);
    float* scores = reinterpret_cast<float*>(ws + L.off_scores);
    uint32_t* bits = reinterpret_cast<uint32_t*>(ws + L.off_bits);
    int32_t* nsel = reinterpret_cast<int32_t*>(ws + L.off_nsel);
    const double scale = params->softmax_scale > 0.f ? (double)params->softmax_scale
                                                     : 1.0 / sqrt((double)params->head_dim);
    const bool use_mma = params->dtype == SPLA_BF16;
    const size_t smem = use_mma ? mma_smem_for(v.d, v.bs, L.max_per)
                                : simt_smem_for(v.d, v.bs, L.max_per);
    if (smem > (size_t)kMaxSmem) return SPLA_ERR_CAPACITY;
    cudaError_t e = launch_shard_mark(v, scores, L.ld, cand_all, nshards, params->top_k,
                                      params->n_sink, params->n_local, first_block, global_nb,
                                      bits, L.nw, nsel, s);
    if (e != cudaSuccess) return cuda_fail(e);
    DecodeArgs da;
    da.q = q;
    da.gamma = nullptr;
    da.out = nullptr;
    da.o_sp = nullptr;
    da.o_rl = nullptr;
    da.bits = bits;
    da.nsel = nsel;
    da.part = reinterpret_cast<float*>(ws + L.off_part);
    da.gread = reinterpret_cast<float*>(ws + L.off_gread);
    da.aw = reinterpret_cast<float*>(ws + L.off_aw);
    da.stamps = nullptr;
    da.status = dev_status;
    da.nw = L.nw;
    da.nsplit = L.nsplit;
    da.max_per = L.max_per;
    da.no_rla = (params->flags & SPLA_FLAG_NO_RLA) ? 1 : 0;
    da.nrd = L.readout_parts;
    da.sl2 = (float)(scale * 1.4426950408889634);
    da.eps = params->rms_eps > 0.f ? params->rms_eps : 1e-6f;
    if (use_mma) {
        CUtensorMap tk, tv;
        if (!make_pool_map(&tk, v.k_pool, v) || !make_pool_map(&tv, v.v_pool, v))
            return cuda_fail(cudaErrorInvalidValue);
        e = launch_decode_mma(v, tk, tv, da, s);
    } else {
        e = launch_decode_simt(v, params->dtype, da, s);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    e = launch_shard_partial(v, params->dtype, da, q, part, s);
    return e == cudaSuccess ? SPLA_OK : cuda_fail(e);
}

spla_status spla_shard_merge(const spla_params* params, int32_t batch, const double* part_all,
                             int32_t nshards, const float* rms_gamma, void* out,
                             float* o_sparse_dbg, float* o_rla_dbg, int32_t* dev_status,
                             void* stream) {
    spla_status st = check_params(params);
    if (st != SPLA_OK) return st;
    if (batch <= 0 || nshards < 1 || !part_all || !out) return SPLA_ERR_INVALID_ARG;
    const float eps = params->rms_eps > 0.f ? params->rms_eps : 1e-6f;
    const int no_rla = (params->flags & SPLA_FLAG_NO_RLA) ? 1 : 0;
    cudaError_t e = launch_shard_merge(batch * params->num_q_heads, params->num_q_heads,
                                       params->head_dim, params->dtype, part_all, nshards, no_rla,
                                       eps, rms_gamma, out, o_sparse_dbg, o_rla_dbg, dev_status,
                                       (cudaStream_t)stream);
    return e == cudaSuccess ? SPLA_OK : cuda_fail(e);
}


// ------------------------------------------------------------------ block-causal form
static spla_status check_block_causal(const spla_params* params, int32_t batch, int32_t max_len) {
    spla_status st = check_params(params);
    if (st != SPLA_OK) return st;
    if (params->dtype != SPLA_BF16 || params->head_dim != 128 ||
        params->num_q_heads / params->num_kv_heads > 4)
        return SPLA_ERR_UNSUPPORTED;
    if (batch <= 0 || max_len <= 0) return SPLA_ERR_INVALID_ARG;
    if ((max_len + params->block_size - 1) / params->block_size > bc_max_blocks() ||
        params->top_k > bc_max_top_k() || (int64_t)batch * max_len > INT32_MAX)
        return SPLA_ERR_CAPACITY;
    return SPLA_OK;
}

spla_status spla_block_causal_workspace_size(const spla_params* params, int32_t batch,
                                             int32_t max_len, size_t* bytes) {
    spla_status st = check_block_causal(params, batch, max_len);
    if (st != SPLA_OK) return st;
    if (!bytes) return SPLA_ERR_INVALID_ARG;
    *bytes = bc_workspace_bytes(batch, params->num_kv_heads, params->block_size, max_len);
    return SPLA_OK;
}

spla_status spla_block_causal_forward(const spla_params* params, const spla_cache* cache,
                                      const void* k_all, const void* v_all, const void* q_all,
                                      int32_t max_len, const float* rms_gamma, void* out,
                                      float* o_sparse_dbg, float* o_rla_dbg, void* workspace,
                                      size_t workspace_bytes, int32_t* dev_status, void* stream) {
    spla_status st = check_params(params);
    if (st != SPLA_OK) return st;
    if ((st = check_cache(cache)) != SPLA_OK) return st;
    if ((st = check_block_causal(params, cache->batch, max_len)) != SPLA_OK) return st;
    if (!k_all || !v_all || !q_all || !out) return SPLA_ERR_INVALID_ARG;
    auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) != 0; };
    if (misaligned(k_all) || misaligned(v_all) || misaligned(q_all) || !cache_aligned(cache) ||
        misaligned(cache->blk_stats) || misaligned(cache->m))
        return SPLA_ERR_INVALID_ARG;
    if ((max_len + params->block_size - 1) / params->block_size > cache->max_blocks_per_seq)
        return SPLA_ERR_CAPACITY;
    const size_t need = bc_workspace_bytes(cache->batch, params->num_kv_heads, params->block_size,
                                           max_len);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return SPLA_ERR_WORKSPACE;
    const CacheView v = view_of(params, cache);
    CUtensorMap tk, tv;
    if (!make_input_map(&tk, k_all, v, max_len) || !make_input_map(&tv, v_all, v, max_len))
        return SPLA_ERR_UNSUPPORTED;
    const double scale = params->softmax_scale > 0.f ? (double)params->softmax_scale
                                                     : 1.0 / sqrt((double)params->head_dim);
    const float eps = params->rms_eps > 0.f ? params->rms_eps : 1e-6f;
    cudaError_t e = launch_block_causal_entry(
        v, tk, tv, k_all, max_len, q_all, rms_gamma, out, o_sparse_dbg, o_rla_dbg, params->top_k,
        params->n_sink, (params->flags & SPLA_FLAG_FIRST_ORDER) ? 1 : 0,
        (params->flags & SPLA_FLAG_NO_RLA) ? 1 : 0, scale, eps, static_cast<char*>(workspace),
        dev_status, (cudaStream_t)stream);
    return e == cudaSuccess ? SPLA_OK : cuda_fail(e);
}

}  // extern "C"
