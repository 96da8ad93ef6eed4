// Context-sharded decode: one long sequence's blocks spread over several GPUs (or
// several caches), each holding a contiguous range of global blocks with their
// statistics and the linear-attention state of its own tokens. The decode step
// of the method (SPLA technical summary, gist.science: section 2.1 selection of
// the blocks with the largest estimates, section 2.2 the residual by
// subtraction, section 2.3 the RMS-normalised output) splits into three phases
// with an exchange between them:
//
//   candidates  per shard: block scores (the scoring kernel), the shard's best
//               top_k + n_sink + n_local blocks (the selection kernel, nothing
//               forced), and from them its best top_k that are not sink or local
//               blocks of the whole sequence, as (score, global block) pairs;
//   -- all-gather of the candidates (top_k pairs per query head and shard) --
//   partials    per shard: the global top-k of the gathered candidates (score
//               descending, ties to the lower global block) fixes a threshold;
//               the shard keeps its forced blocks and every block at or above the
//               threshold, runs the split-KV decode over them, and reduces the
//               splits to one record per head: the softmax state (max m, sum l,
//               unnormalised acc), the residual's numerator N - N~ and
//               denominator D - D~ in fp64 with the log-scale c of the shard's
//               feature weights, and its kept / total block counts;
//   -- all-gather of the records (a few KB per head) --
//   merge       every rank: log-sum-exp merge of the softmax parts, the residual
//               parts rescaled to a common c and added, the subtraction, RMSNorm
//               and the output.
//
// The global top-k is the top-k of the union of every shard's local top-k (a
// block of the global top-k is in its shard's top-k), so the kept set is the one
// an unsharded decode keeps, and every term of the output is a sum over blocks
// or tokens that the shards split without overlap.
#include "common.cuh"

namespace spla {

// A candidate: the block's score and its global index (-1: none).
struct ShardCand {
    float score;
    int32_t block;
};

// Record of one query head from one shard (fp64): [0] m (log2 units), [1] l,
// [2] c, [3] D - D~, [4] kept blocks, [5] blocks, [6] tokens, [7] unused, then
// acc[d] (unnormalised, at m), then N - N~ [d].
__host__ __device__ constexpr int shard_rec_doubles(int d) { return 8 + 2 * d; }

// Composite order of a candidate: larger score first, then lower global block.
__device__ __forceinline__ unsigned long long cand_key(float score, int32_t block) {
    return ((unsigned long long)ordered_key(score) << 32) | (uint32_t)~(uint32_t)block;
}

__device__ __forceinline__ bool forced_block(int32_t gj, int32_t gnb, int n_sink, int n_local) {
    return gj < n_sink || gj >= gnb - n_local;
}

// ------------------------------------------------------------------ candidates
// One warp per (sequence, query head): the blocks the selection kernel kept
// (bitset), minus the sequence's sink and local blocks, ranked; the best top_k
// written in rank order, the rest of the row padded with block -1.
constexpr int kShardCandCap = 1024;

__global__ void __launch_bounds__(32) shard_cand_kernel(CacheView c, const float* scores, int ld,
                                                        const uint32_t* bits, int nw, int top_k,
                                                        int n_sink, int n_local,
                                                        int32_t first_block,
                                                        const int32_t* global_nb,
                                                        ShardCand* cand, int32_t* status) {
    __shared__ unsigned long long ck[kShardCandCap];
    const int head = blockIdx.x;
    const int b = head / c.hq;
    const int lane = threadIdx.x;
    pdl_trigger();
    pdl_wait();
    int32_t L = c.lens[b];
    L = max(0, min(L, c.mbp * c.bs));
    const int nb = (L + c.bs - 1) / c.bs;
    const int32_t gnb = global_nb[b];
    const float* sc = scores + (int64_t)head * ld;
    const uint32_t* hb = bits + (int64_t)head * nw;
    int nc = 0;
    for (int j0 = 0; j0 < nb; j0 += 32) {
        const int j = j0 + lane;
        bool in = false;
        float s = 0.f;
        if (j < nb && ((hb[j0 >> 5] >> lane) & 1u) && !forced_block(first_block + j, gnb, n_sink, n_local)) {
            in = true;
            s = sc[j];
        }
        const uint32_t m = __ballot_sync(0xffffffffu, in);
        if (in) {
            const int p = nc + __popc(m & ((1u << lane) - 1u));
            if (p < kShardCandCap) ck[p] = cand_key(s, first_block + j);
        }
        nc += __popc(m);
    }
    if (nc > kShardCandCap) {
        if (lane == 0) set_status(status, SPLA_DEV_CAPACITY);
        nc = kShardCandCap;
    }
    __syncwarp();
    ShardCand* out = cand + (int64_t)head * top_k;
    for (int i = lane; i < nc; i += 32) {
        const unsigned long long mine = ck[i];
        int rank = 0;
        for (int o = 0; o < nc; ++o) rank += ck[o] > mine;
        if (rank < top_k) {
            ShardCand r;
            r.block = (int32_t)~(uint32_t)mine;
            r.score = sc[r.block - first_block];
            out[rank] = r;
        }
    }
    for (int r = nc + lane; r < top_k; r += 32) {
        ShardCand e;
        e.score = 0.f;
        e.block = -1;
        out[r] = e;
    }
}

// ------------------------------------------------------------------ kept set
// One CTA per (sequence, query head): the top_k-th best of the gathered
// candidates is the threshold; this shard keeps its forced blocks and every
// block at or above it (all blocks when fewer than top_k candidates exist in the
// whole sequence). Writes the head's bitset row (one ballot per 32 blocks) and
// its kept count.
constexpr int kShardMarkThreads = 256;
constexpr int kShardMaxGathered = 4096;

__global__ void __launch_bounds__(kShardMarkThreads)
shard_mark_kernel(CacheView c, const float* scores, int ld, const ShardCand* cand_all,
                  int nshards, int top_k, int n_sink, int n_local, int32_t first_block,
                  const int32_t* global_nb, uint32_t* bits, int nw, int32_t* nsel) {
    __shared__ unsigned long long ck[kShardMaxGathered];
    __shared__ unsigned long long s_thr;
    __shared__ int s_valid, s_kept;
    const int head = blockIdx.x;
    const int b = head / c.hq;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int heads = c.batch * c.hq;
    const int ng = nshards * top_k;
    if (tid == 0) { s_valid = 0; s_kept = 0; s_thr = 0ull; }
    pdl_trigger();
    pdl_wait();
    __syncthreads();
    int valid = 0;
    for (int i = tid; i < ng; i += kShardMarkThreads) {
        const int sh = i / top_k, r = i % top_k;
        const ShardCand e = cand_all[((int64_t)sh * heads + head) * top_k + r];
        const bool ok = e.block >= 0;
        ck[i] = ok ? cand_key(e.score, e.block) : 0ull;
        valid += ok;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) valid += __shfl_xor_sync(0xffffffffu, valid, o);
    if (lane == 0) atomicAdd(&s_valid, valid);
    __syncthreads();
    const bool all_kept = s_valid < top_k;
    if (!all_kept) {
        // the candidate with exactly top_k - 1 better ones (valid keys are distinct)
        for (int i = tid; i < ng; i += kShardMarkThreads) {
            const unsigned long long mine = ck[i];
            if (!mine) continue;
            int rank = 0;
            for (int o = 0; o < ng; ++o) rank += ck[o] > mine;
            if (rank == top_k - 1) s_thr = mine;
        }
    }
    __syncthreads();
    const unsigned long long thr = s_thr;
    int32_t L = c.lens[b];
    L = max(0, min(L, c.mbp * c.bs));
    const int nb = (L + c.bs - 1) / c.bs;
    const int32_t gnb = global_nb[b];
    const float* sc = scores + (int64_t)head * ld;
    uint32_t* hb = bits + (int64_t)head * nw;
    int kept = 0;
    for (int j0 = warp * 32; j0 < nb; j0 += kShardMarkThreads) {
        const int j = j0 + lane;
        bool keep = false;
        if (j < nb) {
            const int32_t gj = first_block + j;
            keep = all_kept || forced_block(gj, gnb, n_sink, n_local) ||
                   cand_key(sc[j], gj) >= thr;
        }
        const uint32_t word = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) hb[j0 >> 5] = word;
        kept += __popc(word);
    }
    if (lane == 0) atomicAdd(&s_kept, kept);
    __syncthreads();
    if (tid == 0) nsel[head] = s_kept;
}

// ------------------------------------------------------------------ per-shard record
// One CTA of 16 warps per (sequence, query head), the split merge of the combine
// step without its last part: the record keeps the softmax state unnormalised and
// the residual as numerator and denominator, with the log-scale c of this shard's
// feature weights a_i = exp(q_i + m_i - c) (c = max_i (q_i + m_i), as the
// scoring kernel forms it).
constexpr int kShardPartThreads = 512;
constexpr int kShardPartWarps = kShardPartThreads / 32;

template <int D, typename T>
__global__ void __launch_bounds__(kShardPartThreads)
shard_partial_kernel(CacheView c, const DecodeArgs a, const T* q, double* rec_out) {
    constexpr int REC = 2 * D + 4;
    const int G = c.group, ns = a.nsplit;
    const int head = blockIdx.x;
    const int b = head / c.hq, hq = head % c.hq;
    const int h = hq / G, g = hq % G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ float s_M, s_l;
    __shared__ double s_dt;
    __shared__ float s_cw[kShardPartWarps];
    __shared__ float s_po[kShardPartWarps][D];
    __shared__ double s_pn[kShardPartWarps][D];
    extern __shared__ __align__(16) float smem_sp[];   // [ns][4] headers
    float* hdr = smem_sp;
    pdl_wait();
    const float* recs = a.part + (((int64_t)b * c.hkv + h) * ns * G + g) * REC;
    const float* gr = a.gread + (((int64_t)b * c.hkv + h) * a.nrd * G + g) * (D + 4);
    for (int s = tid; s < ns; s += kShardPartThreads)
        reinterpret_cast<float4*>(hdr)[s] =
            __ldcg(reinterpret_cast<const float4*>(recs + (int64_t)s * G * REC));
    // readout and the scale c: thread i < D owns dimension i
    double Nj = 0.0, Dg = 0.0;
    float cv = -SPLA_INF;
    if (tid < D) {
        for (int p = 0; p < a.nrd; ++p) {
            Nj += (double)__ldcg(gr + (int64_t)p * G * (D + 4) + tid);
            if (tid == 0) Dg += (double)__ldcg(gr + (int64_t)p * G * (D + 4) + D);
        }
        const int64_t gi = (int64_t)b * c.hkv + h;
        cv = to_f(q[((int64_t)b * c.hq + hq) * D + tid]) + c.m[gi * D + tid];
    }
    cv = warp_max(cv);
    if (lane == 0) s_cw[warp] = cv;
    __syncthreads();
    if (warp == 0) {
        float M = -SPLA_INF;
        for (int s = lane; s < ns; s += 32) M = fmaxf(M, hdr[4 * s]);
        M = warp_max(M);
        float l = 0.f;
        double dt = 0.0;
        for (int s = lane; s < ns; s += 32) {
            const float f = (M == -SPLA_INF) ? 0.f : ex2(hdr[4 * s] - M);
            hdr[4 * s + 3] = f;                 // the split's factor, in the unused slot
            l += hdr[4 * s + 1] * f;
            dt += (double)hdr[4 * s + 2];
        }
        l = warp_sum(l);
#pragma unroll
        for (int o = 16; o; o >>= 1) dt += __shfl_xor_sync(0xffffffffu, dt, o);
        if (lane == 0) { s_M = M; s_l = l; s_dt = dt; }
    }
    __syncthreads();
    constexpr int CPL = D / 32;
    float o[CPL];
    double nt[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) { o[e] = 0.f; nt[e] = 0.0; }
    for (int s = warp; s < ns; s += kShardPartWarps) {
        const float* r = recs + (int64_t)s * G * REC + 4 + lane * CPL;
        const float f = hdr[4 * s + 3];
#pragma unroll
        for (int e = 0; e < CPL; ++e) {
            o[e] = fmaf(__ldcg(r + e), f, o[e]);
            nt[e] += (double)__ldcg(r + D + e);
        }
    }
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
        s_po[warp][lane * CPL + e] = o[e];
        s_pn[warp][lane * CPL + e] = nt[e];
    }
    __syncthreads();
    double* out = rec_out + (int64_t)head * shard_rec_doubles(D);
    if (tid < D) {
        float ot = 0.f;
        double ntt = 0.0;
#pragma unroll
        for (int w = 0; w < kShardPartWarps; ++w) {
            ot += s_po[w][tid];
            ntt += s_pn[w][tid];
        }
        out[8 + tid] = (double)ot;
        out[8 + D + tid] = Nj - ntt;
    }
    if (tid == 0) {
        float cmax = -SPLA_INF;
        for (int w = 0; w < D / 32; ++w) cmax = fmaxf(cmax, s_cw[w]);
        int32_t L = c.lens[b];
        L = max(0, min(L, c.mbp * c.bs));
        out[0] = (double)s_M;
        out[1] = (double)s_l;
        out[2] = (double)cmax;
        out[3] = Dg - s_dt;
        out[4] = (double)a.nsel[head];
        out[5] = (double)((L + c.bs - 1) / c.bs);
        out[6] = (double)L;
        out[7] = 0.0;
    }
}

// ------------------------------------------------------------------ merge
// One warp per (sequence, query head), lane l holding columns [l d/32, (l+1) d/32):
// log-sum-exp merge of the shards' softmax parts, their residual parts rescaled
// by exp(c_s - C) (C the largest c of a shard holding tokens) and added, the
// subtraction, RMSNorm and the output. Lane s reads shard s's header (shards
// past 32 in further rounds), so the maxima need one round trip; the records'
// columns follow, four shards' loads in flight at a time.
constexpr int kShardMergeWarps = 1;
constexpr int kShardMergeBatch = 4;

template <int D, typename T>
__global__ void __launch_bounds__(kShardMergeWarps * 32)
shard_merge_kernel(int heads, int hq_count, const double* rec_all, int nshards, int no_rla,
                   float eps, const float* gamma, T* out, float* o_sp, float* o_rl,
                   int32_t* status) {
    constexpr int CPL = D / 32;
    constexpr int R = shard_rec_doubles(D);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int head = blockIdx.x * kShardMergeWarps + warp;
    pdl_wait();
    if (head >= heads) return;
    const int hq = head % hq_count;
    auto rec = [&](int s) { return rec_all + ((int64_t)s * heads + head) * R; };
    double M = -INFINITY, C = -INFINITY, kept = 0.0, nblk = 0.0, ntok = 0.0;
    for (int s = lane; s < nshards; s += 32) {
        const double* r = rec(s);
        const double m = r[0], cc = r[2], kk = r[4], nb = r[5], nt = r[6];
        M = fmax(M, m);
        if (nt > 0.0) C = fmax(C, cc);
        kept += kk;
        nblk += nb;
        ntok += nt;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        M = fmax(M, __shfl_xor_sync(0xffffffffu, M, o));
        C = fmax(C, __shfl_xor_sync(0xffffffffu, C, o));
        kept += __shfl_xor_sync(0xffffffffu, kept, o);
        nblk += __shfl_xor_sync(0xffffffffu, nblk, o);
        ntok += __shfl_xor_sync(0xffffffffu, ntok, o);
    }
    double l = 0.0, rD = 0.0, o[CPL], rN[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) { o[e] = 0.0; rN[e] = 0.0; }
    for (int s0 = 0; s0 < nshards; s0 += kShardMergeBatch) {
        double hm[kShardMergeBatch], hl[kShardMergeBatch], hc[kShardMergeBatch],
            hd[kShardMergeBatch], ht[kShardMergeBatch];
        double xo[kShardMergeBatch][CPL], xn[kShardMergeBatch][CPL];
#pragma unroll
        for (int u = 0; u < kShardMergeBatch; ++u) {
            if (s0 + u < nshards) {
                const double* r = rec(s0 + u);
                hm[u] = r[0]; hl[u] = r[1]; hc[u] = r[2]; hd[u] = r[3]; ht[u] = r[6];
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    xo[u][e] = r[8 + lane * CPL + e];
                    xn[u][e] = r[8 + D + lane * CPL + e];
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kShardMergeBatch; ++u) {
            if (s0 + u < nshards) {
                const double f = (M == -INFINITY || hm[u] == -INFINITY) ? 0.0 : exp2(hm[u] - M);
                const double w = (ht[u] > 0.0 && C != -INFINITY) ? exp(hc[u] - C) : 0.0;
                l += hl[u] * f;
                rD += hd[u] * w;
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    o[e] += xo[u][e] * f;
                    rN[e] += xn[u][e] * w;
                }
            }
        }
    }
    const bool off = no_rla || kept >= nblk || ntok == 0.0;
    const bool unresolved = !off && !(rD > 0.0);
    if (unresolved && lane == 0) set_status(status, SPLA_DEV_RLA_UNRESOLVED);
    float osp[CPL], orl[CPL], sq = 0.f;
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
        osp[e] = (l > 0.0) ? (float)(o[e] / l) : 0.f;
        orl[e] = (off || unresolved) ? 0.f : (float)(rN[e] / rD);
        sq = fmaf(orl[e], orl[e], sq);
    }
    sq = warp_sum(sq);
    const float inv = rsqrtf(sq / D + eps);
    const int64_t o0 = (int64_t)head * D + lane * CPL;
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
        const float gm = gamma ? gamma[(int64_t)hq * D + lane * CPL + e] : 1.f;
        out[o0 + e] = from_f<T>(osp[e] + gm * orl[e] * inv);
        if (o_sp) o_sp[o0 + e] = osp[e];
        if (o_rl) o_rl[o0 + e] = orl[e];
    }
}

// ------------------------------------------------------------------ launchers
int shard_max_gathered() { return kShardMaxGathered; }

cudaError_t launch_shard_cand(const CacheView& c, const float* scores, int ld,
                              const uint32_t* bits, int nw, int top_k, int n_sink, int n_local,
                              int32_t first_block, const int32_t* global_nb, void* cand,
                              int32_t* status, cudaStream_t s) {
    return launch_pdl(shard_cand_kernel, dim3(c.batch * c.hq), dim3(32), 0, s, c, scores, ld, bits,
                      nw, top_k, n_sink, n_local, first_block, global_nb,
                      static_cast<ShardCand*>(cand), status);
}

cudaError_t launch_shard_mark(const CacheView& c, const float* scores, int ld,
                              const void* cand_all, int nshards, int top_k, int n_sink,
                              int n_local, int32_t first_block, const int32_t* global_nb,
                              uint32_t* bits, int nw, int32_t* nsel, cudaStream_t s) {
    return launch_pdl(shard_mark_kernel, dim3(c.batch * c.hq), dim3(kShardMarkThreads), 0, s, c,
                      scores, ld, static_cast<const ShardCand*>(cand_all), nshards, top_k, n_sink,
                      n_local, first_block, global_nb, bits, nw, nsel);
}

cudaError_t launch_shard_partial(const CacheView& c, int dtype, const DecodeArgs& a,
                                 const void* q, double* rec, cudaStream_t s) {
    const size_t smem = (size_t)4 * a.nsplit * sizeof(float);
    const dim3 grid(c.batch * c.hq), block(kShardPartThreads);
    using B16 = __nv_bfloat16;
    if (c.d == 128)
        return dtype == SPLA_BF16
            ? launch_pdl(shard_partial_kernel<128, B16>, grid, block, smem, s, c, a, (const B16*)q, rec)
            : launch_pdl(shard_partial_kernel<128, float>, grid, block, smem, s, c, a, (const float*)q, rec);
    return dtype == SPLA_BF16
        ? launch_pdl(shard_partial_kernel<64, B16>, grid, block, smem, s, c, a, (const B16*)q, rec)
        : launch_pdl(shard_partial_kernel<64, float>, grid, block, smem, s, c, a, (const float*)q, rec);
}

cudaError_t launch_shard_merge(int heads, int hq, int d, int dtype, const double* rec_all,
                               int nshards, int no_rla, float eps, const float* gamma, void* out,
                               float* o_sp, float* o_rl, int32_t* status, cudaStream_t s) {
    const dim3 grid((heads + kShardMergeWarps - 1) / kShardMergeWarps), block(kShardMergeWarps * 32);
    using B16 = __nv_bfloat16;
    if (d == 128)
        return dtype == SPLA_BF16
            ? launch_pdl(shard_merge_kernel<128, B16>, grid, block, 0, s, heads, hq, rec_all, nshards,
                         no_rla, eps, gamma, (B16*)out, o_sp, o_rl, status)
            : launch_pdl(shard_merge_kernel<128, float>, grid, block, 0, s, heads, hq, rec_all,
                         nshards, no_rla, eps, gamma, (float*)out, o_sp, o_rl, status);
    return dtype == SPLA_BF16
        ? launch_pdl(shard_merge_kernel<64, B16>, grid, block, 0, s, heads, hq, rec_all, nshards,
                     no_rla, eps, gamma, (B16*)out, o_sp, o_rl, status)
        : launch_pdl(shard_merge_kernel<64, float>, grid, block, 0, s, heads, hq, rec_all, nshards,
                     no_rla, eps, gamma, (float*)out, o_sp, o_rl, status);
}

}  // namespace spla
