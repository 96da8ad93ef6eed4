// a3 + a4 + a5 -- split-KV decode over the kept blocks with the residual linear
// attention computed in the same pass, and the split combine (SPLA technical
// summary, gist.science: section 2 opening -- exact attention over the kept
// blocks; section 2.2 -- RLA by subtraction, the kept blocks' linear-attention
// term computed while they are on chip so unkept blocks are never read;
// section 2.3 -- exponential feature map, RMS-normalised RLA added to the
// sparse output). Softmax is softmax(q k^T / sqrt(d)) as in the Baidu article
// "Sparse Attention for Long-Context LLMs: Implementation and Trade-off
// Design", section 1; normalised linear attention as in its section 7.
//
// Grid (nsplit, batch*Hkv). Every CTA of a (sequence, KV head) group:
//   * forms the union of the G heads' selections from their bitsets (all
//     threads, one block scan over the words) and takes an equal share of it
//     (a union block is read once for all G heads; a head that did not select
//     it is masked out of it);
//   * streams its blocks' K and V tiles and accumulates, per head, the online
//     softmax (m, l, acc = sum p v) and the kept blocks' linear-attention
//     numerator and denominator (N~ = sum w v, D~ = sum w) with
//     w_t = sum_i exp(q_i + m_i - c) exp(k_t,i - m_i);
//   * writes one partial record per head: m, l, acc, N~, D~.
// combine_kernel (one CTA of 16 warps per query head, launched right behind)
// merges the head's records: log-sum-exp merge of the softmax partials,
// o_rla = (N - N~)/(D - D~) with the global readout N, D the scoring kernel
// computed from S, z (the kept blocks' N~, D~ and the subtraction in fp64);
// RMSNorm; out = o_sparse + gamma * RMSNorm(o_rla).
//
// decode_mma_kernel (bf16 K/V): 4 consumer warps + 1 TMA producer warp, three
// CTAs per SM (128 registers). The pipeline unit is a 64-token tile of one
// (block, KV head): its K and V come by 2-D tiled TMA (128-byte swizzle, no
// multicast) into a 2-deep mbarrier ring per CTA, so six units per SM are in
// flight (a 128-token block is two units). Each consumer warp
// owns one 16-token slab of a unit and runs the G-head contractions on tensor
// cores (mma.sync m16n8k16 bf16, fp32 accumulate):
//   logits  = K(16 x d) . Q^T(d x 8)            (q exact in bf16)
//   w       = phi(K)(16 x d) . [a_hi a_lo]^T    (phi(K) split hi/lo in bf16)
//   O^T    += V^T(d x 16) . [P W]_{hi,lo}       (P, W split hi/lo in bf16)
// so every computed operand carries ~16 mantissa bits.
// decode_simt_kernel (fp32 or bf16 K/V): plain fp32 FMA, for the fp32 path.
#include "common.cuh"

namespace spla {

// ------------------------------------------------------------------ shared prologue pieces
// Query-side constants, loaded before the dependency wait (inputs and what the
// append and scoring kernels wrote): qs[g][i] = q (fp32), ml[i] = m_i * log2e
// and the phi weights aw[g][i] = exp(q_g,i + m_i - c_g) the scoring kernel used
// for the global readout (the kept blocks' term uses the very same weights).
// With trow non-null, also the sequence's block-table row (mbp entries).
// (Out of line, scalar arguments: the prologue does not add to the register
// pressure of the streaming loop that follows it.)
__device__ __noinline__ void stage_query(const void* q, const float* aw_ws, const float* m,
                                         const int32_t* table, int mbp, int hq, int hkv, int G,
                                         int d, int is_bf16, int b, int h, float* qs, float* ml,
                                         float* aw, int32_t* trow, int tid, int nthr) {
    const int gi = b * hkv + h;
    const float* mrow = m + (int64_t)gi * d;
    for (int e = tid; e < G * d; e += nthr) {
        const int g = e / d, i = e % d;
        const int64_t qi = ((int64_t)b * hq + h * G + g) * d + i;
        qs[e] = is_bf16 ? __bfloat162float(((const __nv_bfloat16*)q)[qi]) : ((const float*)q)[qi];
        aw[e] = __ldcg(aw_ws + ((int64_t)gi * d + i) * 4 + g);
    }
    for (int i = tid; i < d; i += nthr) ml[i] = mrow[i] * SPLA_LOG2E;
    if (trow) {
        const int32_t* src = table + (int64_t)b * mbp;
        for (int j = tid; j < mbp; j += nthr) trow[j] = __ldcg(src + j);
    }
}

// Tensor-core path, before the dependency wait, one round of 16-byte loads (all
// issued before any shared-memory store): the group's G query rows as raw bf16
// (qraw[g][d]), the phi weights aw[i][4] = exp(q_g,i + m_i - c_g) the scoring
// kernel used for the global readout (the kept blocks' term uses the very same
// weights), m_i * log2e (ml[d]) and, with trow non-null, the sequence's
// block-table row (its entry j at trow[j]). (Out of line, scalar arguments: the
// prologue does not add to the register pressure of the streaming loop.)
__device__ __noinline__ void stage_query_vec(const __nv_bfloat16* q, const float* aw_ws,
                                             const float* m, const int32_t* table, int mbp,
                                             int hq, int hkv, int G, int d, int b, int h,
                                             uint32_t* qraw, float* aw, float* ml,
                                             int32_t* trow_area, int32_t** trow, int tid,
                                             int nthr) {
    const int gi = b * hkv + h;
    const int4* srcq = reinterpret_cast<const int4*>(q + ((int64_t)b * hq + h * G) * d);
    const int4* srca = reinterpret_cast<const int4*>(aw_ws + (int64_t)gi * d * 4);
    const int4* srcm = reinterpret_cast<const int4*>(m + (int64_t)gi * d);
    const int nq = G * d / 8, na = d, nm = d / 4;            // int4 counts
    // the table row: from the 16-byte boundary at or before its start; whole int4
    // chunks that end inside the row, then the last few entries one by one
    const int32_t* row = table + (int64_t)b * mbp;
    const int off = trow_area ? (int)((reinterpret_cast<uintptr_t>(row) & 15) >> 2) : 0;
    const int4* srct = reinterpret_cast<const int4*>(row - off);
    const int nt = trow_area ? (off + mbp) / 4 : 0;
    const int total = nq + na + nm + nt;
    constexpr int kBatch = 8;
    for (int e0 = tid; e0 < total; e0 += kBatch * nthr) {
        int4 v[kBatch];
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int e = e0 + k * nthr;
            if (e < nq) v[k] = __ldg(srcq + e);
            else if (e < nq + na) v[k] = __ldcg(srca + (e - nq));
            else if (e < nq + na + nm) v[k] = __ldcg(srcm + (e - nq - na));
            else if (e < total) v[k] = __ldcg(srct + (e - nq - na - nm));
        }
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int e = e0 + k * nthr;
            if (e < nq) reinterpret_cast<int4*>(qraw)[e] = v[k];
            else if (e < nq + na) reinterpret_cast<int4*>(aw)[e - nq] = v[k];
            else if (e < nq + na + nm) {
                const int4 x = v[k];
                float4 f = make_float4(__int_as_float(x.x) * SPLA_LOG2E, __int_as_float(x.y) * SPLA_LOG2E,
                                       __int_as_float(x.z) * SPLA_LOG2E, __int_as_float(x.w) * SPLA_LOG2E);
                reinterpret_cast<float4*>(ml)[e - nq - na] = f;
            } else if (e < total) {
                reinterpret_cast<int4*>(trow_area)[e - nq - na - nm] = v[k];
            }
        }
    }
    if (trow_area) {
        for (int j = nt * 4 + tid; j < off + mbp; j += nthr) trow_area[j] = __ldcg(row - off + j);
        *trow = trow_area + off;
    }
}

// After the wait, one round of 16-byte loads: the G heads' selection bitset rows
// (stride nw, a multiple of 4 words) into wbits[G][nw].
__device__ __noinline__ void stage_bits_vec(const uint32_t* bits, int nw, int hq, int G, int b,
                                            int h, uint32_t* wbits, int tid, int nthr) {
    const int4* src = reinterpret_cast<const int4*>(bits + ((int64_t)b * hq + h * G) * nw);
    const int n4 = G * nw / 4;
    constexpr int kBatch = 4;
    for (int e0 = tid; e0 < n4; e0 += kBatch * nthr) {
        int4 v[kBatch];
#pragma unroll
        for (int k = 0; k < kBatch; ++k)
            if (e0 + k * nthr < n4) v[k] = __ldcg(src + e0 + k * nthr);
#pragma unroll
        for (int k = 0; k < kBatch; ++k)
            if (e0 + k * nthr < n4) reinterpret_cast<int4*>(wbits)[e0 + k * nthr] = v[k];
    }
}

// After the wait, one round of loads: the G heads' selection bitset words of
// this group into wbits ([G][nwu], shared memory).
__device__ __forceinline__ void stage_bits(const uint32_t* bits, int nw, int hq, int G, int b,
                                           int h, int nwu, uint32_t* wbits, int tid, int nthr) {
    const uint32_t* hb = bits + ((int64_t)b * hq + h * G) * nw;
    for (int e = tid; e < G * nwu; e += nthr) {
        const int g = e / nwu, w = e % nwu;
        wbits[e] = __ldcg(hb + (int64_t)g * nw + w);
    }
}

// Then, from shared memory: the union of the G selections (a block read once
// for all heads that kept it), per-word counts and their prefix sums (one
// warp), this CTA's equal share [u0, u1) of the union with per-block head
// masks, and the share's physical blocks from the table row trow (shared or
// global memory). wcnt: nwu ints of scratch. Returns the share's length (all
// threads).
__device__ __noinline__ int union_share(const int32_t* trow, int num_phys, int G,
                                        const uint32_t* wbits, int nwu, int nb, int split,
                                        int nsplit, int max_per, int* wcnt, int32_t* blk,
                                        int32_t* phys, uint32_t* hm, int* s_n, int32_t* status,
                                        int tid, int nthr) {
    const int lane = tid & 31, warp = tid >> 5;
    auto word = [&](int w) -> uint32_t {
        uint32_t u = 0u;
        for (int g = 0; g < G; ++g) u |= wbits[g * nwu + w];
        if (w == nwu - 1 && (nb & 31)) u &= (1u << (nb & 31)) - 1u;
        return u;
    };
    for (int w = tid; w < nwu; w += nthr) wcnt[w] = __popc(word(w));
    __syncthreads();
    if (warp == 0) {
        const int wpl = (nwu + 31) >> 5;
        const int w0 = lane * wpl, w1 = min(nwu, w0 + wpl);
        int cnt = 0;
        for (int w = w0; w < w1; ++w) cnt += wcnt[w];
        int x = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        int run = x - cnt;
        for (int w = w0; w < w1; ++w) {
            const int v = wcnt[w];
            wcnt[w] = run;
            run += v;
        }
        if (lane == 31) {
            s_n[0] = (int)(((int64_t)split * x) / nsplit);          // u0
            s_n[1] = (int)(((int64_t)(split + 1) * x) / nsplit);    // u1
        }
    }
    __syncthreads();
    const int u0 = s_n[0], u1 = s_n[1];
    for (int w = tid; w < nwu; w += nthr) {
        const int base = wcnt[w];
        if (base >= u1) continue;
        uint32_t u = word(w);
        if (base + __popc(u) <= u0) continue;
        int r = base;
        while (u) {
            const int bit = __ffs(u) - 1;
            u &= u - 1u;
            if (r >= u0 && r < u1 && r - u0 < max_per) {
                uint32_t mask = 0u;
                for (int g = 0; g < G; ++g) mask |= ((wbits[g * nwu + w] >> bit) & 1u) << g;
                blk[r - u0] = (w << 5) + bit;
                hm[r - u0] = mask;
            }
            ++r;
        }
    }
    __syncthreads();
    const int n = min(u1 - u0, max_per);
    for (int e = tid; e < n; e += nthr) {
        int32_t p = trow[blk[e]];
        if (p < 0 || p >= num_phys) {
            // read nothing from it: no head attends to it
            set_status(status, SPLA_DEV_BAD_BLOCK_TABLE);
            p = 0;
            hm[e] = 0u;
        }
        phys[e] = p;
    }
    __syncthreads();
    return n;
}

// This CTA's share of the union of the group's G selections, built by all NT
// threads: thread t takes consecutive words [t W, t W + W) so that union ranks run
// in word order; one block scan of the per-thread counts gives every thread its
// first rank, and the ranks in [u0, u1) = [split tot / nsplit, (split+1) tot / nsplit)
// are written out in rank order (block index, head mask, physical block).
// wbits: [G][ws] words in shared memory, the first nwu of each row in use.
template <int NT>
__device__ int union_share_cta(const int32_t* trow, int num_phys, int G, const uint32_t* wbits,
                               int ws, int nwu, int nb, int split, int nsplit, int max_per,
                               int32_t* blk, int32_t* phys, uint32_t* hm, int32_t* status,
                               int* s_wsum) {
    constexpr int NWARP = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto word = [&](int w) -> uint32_t {
        uint32_t u = 0u;
        for (int g = 0; g < G; ++g) u |= wbits[g * ws + w];
        if (w == nwu - 1 && (nb & 31)) u &= (1u << (nb & 31)) - 1u;
        return u;
    };
    const int wpt = (nwu + NT - 1) / NT;
    const int w0 = min(nwu, tid * wpt), w1 = min(nwu, w0 + wpt);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(word(w));
    int x = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_wsum[warp] = x;
    __syncthreads();
    int before = x - cnt, tot = 0;
#pragma unroll
    for (int v = 0; v < NWARP; ++v) {
        const int t = s_wsum[v];
        if (v < warp) before += t;
        tot += t;
    }
    // the union holds at most 32768 blocks and nsplit is at most 512: 32-bit products
    const int u0 = split * tot / nsplit, u1 = (split + 1) * tot / nsplit;
    int r = before;
    for (int w = w0; w < w1 && r < u1; ++w) {
        uint32_t u = word(w);
        const int cw = __popc(u);
        if (r + cw <= u0) { r += cw; continue; }
        while (u) {
            const int bit = __ffs(u) - 1;
            u &= u - 1u;
            if (r >= u0 && r < u1 && r - u0 < max_per) {
                const int e = r - u0, j = (w << 5) + bit;
                uint32_t mask = 0u;
                for (int g = 0; g < G; ++g) mask |= ((wbits[g * ws + w] >> bit) & 1u) << g;
                int32_t p = trow[j];
                if (p < 0 || p >= num_phys) {
                    // read nothing from it: no head attends to it
                    set_status(status, SPLA_DEV_BAD_BLOCK_TABLE);
                    p = 0;
                    mask = 0u;
                }
                blk[e] = j;
                hm[e] = mask;
                phys[e] = p;
            }
            ++r;
        }
    }
    return min(u1 - u0, max_per);
}

// ------------------------------------------------------------------ combine
// One CTA of 16 warps per (sequence, query head). Warp w takes the splits
// w, w + 16, ...: lane l holds columns [l d/32, (l+1) d/32) of their acc and N~
// (vector loads), so up to 64 splits' records are in flight in one round trip
// together with the headers and the readout N, D; the warps' partial sums meet
// in shared memory. Launched right behind the decode kernel (programmatic
// dependent launch), it waits for it.
constexpr int kCombThreads = 512;
constexpr int kCombWarps = kCombThreads / 32;
constexpr int kCombPerWarp = 4;                 // splits per warp per round trip

template <int D> struct CombVec;
template <> struct CombVec<128> {
    static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
        const float4 x = __ldcg(reinterpret_cast<const float4*>(p));
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    }
};
template <> struct CombVec<64> {
    static __device__ __forceinline__ void load(const float* p, float (&v)[2]) {
        const float2 x = __ldcg(reinterpret_cast<const float2*>(p));
        v[0] = x.x; v[1] = x.y;
    }
};

template <int D, typename T>
__global__ void __launch_bounds__(kCombThreads) combine_kernel(CacheView c, const DecodeArgs a) {
    constexpr int CPL = D / 32;                 // columns per lane
    extern __shared__ __align__(16) float smem_comb[];
    const int G = c.group, ns = a.nsplit;
    constexpr int REC = 2 * D + 4;
    const int b = blockIdx.x / c.hq, hq = blockIdx.x % c.hq;
    const int h = hq / G, g = hq % G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float* hdr = smem_comb;                     // [ns][4]: m, l, D~
    float* fac = hdr + 4 * ns;                  // [ns]
    __shared__ __align__(16) float s_po[kCombWarps][D];
    __shared__ __align__(16) double s_pn[kCombWarps][D];
    __shared__ float s_M, s_l, s_red[D / 32];
    __shared__ double s_dt, s_D;
    pdl_wait();
    if (tid == 0) stamp_first(a.stamps, kStampCombine);
    const float* recs = a.part + (((int64_t)b * c.hkv + h) * ns * G + g) * REC;   // split s at s*G*REC
    const float* gr = a.gread + (((int64_t)b * c.hkv + h) * a.nrd * G + g) * (D + 4);
    for (int s = tid; s < ns; s += kCombThreads)
        reinterpret_cast<float4*>(hdr)[s] = __ldcg(reinterpret_cast<const float4*>(recs + (int64_t)s * G * REC));
    // this warp's first splits, in flight with the headers
    float acc[kCombPerWarp][CPL], ntl[kCombPerWarp][CPL];
#pragma unroll
    for (int u = 0; u < kCombPerWarp; ++u) {
        const int s = warp + u * kCombWarps;
#pragma unroll
        for (int e = 0; e < CPL; ++e) acc[u][e] = ntl[u][e] = 0.f;
        if (s < ns) {
            const float* r = recs + (int64_t)s * G * REC + 4 + lane * CPL;
            CombVec<D>::load(r, acc[u]);
            CombVec<D>::load(r + D, ntl[u]);
        }
    }
    double Nj = 0.0, Dg = 0.0;
    if (tid < D)
        for (int p = 0; p < a.nrd; ++p) {          // the readout's row-range parts add
            Nj += (double)__ldcg(gr + (int64_t)p * G * (D + 4) + tid);
            if (tid == 0) Dg += (double)__ldcg(gr + (int64_t)p * G * (D + 4) + D);
        }
    if (tid == 0) s_D = Dg;
    const int nsel = a.nsel[(int64_t)b * c.hq + hq];
    int32_t L = c.lens[b];
    L = max(0, min(L, c.mbp * c.bs));
    const int nb = (L + c.bs - 1) / c.bs;
    __syncthreads();
    if (warp == 0) {
        float M = -SPLA_INF;
        for (int s = lane; s < ns; s += 32) M = fmaxf(M, hdr[4 * s]);
        M = warp_max(M);
        float l = 0.f;
        double dt = 0.0;
        for (int s = lane; s < ns; s += 32) {
            const float f = (M == -SPLA_INF) ? 0.f : ex2(hdr[4 * s] - M);
            fac[s] = f;
            l += hdr[4 * s + 1] * f;
            dt += (double)hdr[4 * s + 2];
        }
        l = warp_sum(l);
#pragma unroll
        for (int o = 16; o; o >>= 1) dt += __shfl_xor_sync(0xffffffffu, dt, o);
        if (lane == 0) { s_M = M; s_l = l; s_dt = dt; }
    }
    __syncthreads();
    float o[CPL];
    double nt[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) { o[e] = 0.f; nt[e] = 0.0; }
#pragma unroll
    for (int u = 0; u < kCombPerWarp; ++u) {
        const int s = warp + u * kCombWarps;
        if (s < ns) {
            const float f = fac[s];
#pragma unroll
            for (int e = 0; e < CPL; ++e) {
                o[e] = fmaf(acc[u][e], f, o[e]);
                nt[e] += (double)ntl[u][e];
            }
        }
    }
    // more than kCombWarps * kCombPerWarp splits: further round trips
    for (int s0 = kCombWarps * kCombPerWarp; s0 < ns; s0 += kCombWarps * kCombPerWarp) {
#pragma unroll
        for (int u = 0; u < kCombPerWarp; ++u) {
            const int s = s0 + warp + u * kCombWarps;
#pragma unroll
            for (int e = 0; e < CPL; ++e) acc[u][e] = ntl[u][e] = 0.f;
            if (s < ns) {
                const float* r = recs + (int64_t)s * G * REC + 4 + lane * CPL;
                CombVec<D>::load(r, acc[u]);
                CombVec<D>::load(r + D, ntl[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < kCombPerWarp; ++u) {
            const int s = s0 + warp + u * kCombWarps;
            if (s < ns) {
                const float f = fac[s];
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    o[e] = fmaf(acc[u][e], f, o[e]);
                    nt[e] += (double)ntl[u][e];
                }
            }
        }
    }
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
        s_po[warp][lane * CPL + e] = o[e];
        s_pn[warp][lane * CPL + e] = nt[e];
    }
    __syncthreads();
    // thread j < D finishes column j
    float osp = 0.f, orl = 0.f;
    if (tid < D) {
        float ot = 0.f;
        double ntt = 0.0;
#pragma unroll
        for (int w = 0; w < kCombWarps; ++w) {
            ot += s_po[w][tid];
            ntt += s_pn[w][tid];
        }
        const float lsum = s_l;
        const double Dr = s_D - s_dt;
        const bool off = a.no_rla || nsel >= nb || L == 0;
        // the residual mass is below what the state resolves: o_rla = 0, and the caller is told
        const bool unresolved = !off && !(Dr > 0.0);
        if (unresolved && tid == 0) set_status(a.status, SPLA_DEV_RLA_UNRESOLVED);
        osp = (lsum > 0.f) ? ot / lsum : 0.f;
        orl = (off || unresolved) ? 0.f : (float)((Nj - ntt) / Dr);
        // RMS of o_rla over the head dimension
        const float sq = warp_sum(orl * orl);
        if (lane == 0) s_red[warp] = sq;
    }
    __syncthreads();
    if (tid < D) {
        float sq = 0.f;
#pragma unroll
        for (int w = 0; w < D / 32; ++w) sq += s_red[w];
        const float inv = rsqrtf(sq / D + a.eps);
        const int64_t oi = ((int64_t)b * c.hq + hq) * D + tid;
        const float gm = a.gamma ? a.gamma[(int64_t)hq * D + tid] : 1.f;
        static_cast<T*>(a.out)[oi] = from_f<T>(osp + gm * orl * inv);
        if (a.o_sp) a.o_sp[oi] = osp;
        if (a.o_rl) a.o_rl[oi] = orl;
    }
    if (tid == 0) stamp_last(a.stamps, kStampCombine);
}

// ------------------------------------------------------------------ bf16 tensor-core kernel
template <int D, int UPB, int STAGES>
struct MmaCfg {
    static constexpr int NCW = 4;                           // consumer warps (one slab each)
    static constexpr int THREADS = (NCW + 1) * 32;
    static constexpr int BS = 64 * UPB;                     // tokens per block
    static constexpr int BOXES = D / 64;                    // 64-column boxes per tile
    static constexpr int BOX_BYTES = 64 * 128;              // 64 rows x 128 B
    static constexpr int TILE_BYTES = BOXES * BOX_BYTES;    // one of K or V for a unit
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
};

template <int D, int UPB, int STAGES>
__global__ void __launch_bounds__(MmaCfg<D, UPB, STAGES>::THREADS, 3)
decode_mma_kernel(const __grid_constant__ CacheView c, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ DecodeArgs a) {
    using Cfg = MmaCfg<D, UPB, STAGES>;
    constexpr int NCW = Cfg::NCW, G4 = 4, BS = Cfg::BS;
    extern __shared__ __align__(1024) unsigned char smem_mma[];
    // carve: stages (1024-aligned) | barriers | lists | query constants
    unsigned char* stages = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_mma) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(stages + STAGES * Cfg::STAGE_BYTES);
    uint64_t* empty = full + STAGES;
    int32_t* blk = reinterpret_cast<int32_t*>(empty + STAGES);
    int32_t* phys = blk + a.max_per;
    uint32_t* hm = reinterpret_cast<uint32_t*>(phys + a.max_per);
    // 16-byte aligned: ml is read as float2 (max_per may be odd)
    float* qs = reinterpret_cast<float*>(
        (reinterpret_cast<uintptr_t>(hm + a.max_per) + 15) & ~uintptr_t(15));   // [4][D]
    float* aw = qs + G4 * D;                                // [4][D]
    float* ml = aw + G4 * D;                                // [D]
    __shared__ int s_n[2], s_abort, s_wsum[Cfg::THREADS / 32];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y / c.hkv, h = blockIdx.y % c.hkv, split = blockIdx.x;
    const int G = c.group, nsplit = a.nsplit;
    pdl_trigger();
    if (tid == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    // Before the dependency wait (the selection kernel launches this one once the
    // scoring kernel has completed): lengths, query constants and the block-table
    // row, which depend only on the append and scoring kernels. The bitset words,
    // counts and table row borrow the stage buffers (no TMA in flight yet).
    int32_t L = c.lens[b];
    if (L < 0 || L > c.mbp * c.bs) L = max(0, min(L, c.mbp * c.bs));
    const int nb = (L + BS - 1) / BS;
    const int64_t rec_base = (((int64_t)b * c.hkv + h) * nsplit + split) * G;
    constexpr int REC = 2 * D + 4;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NCW);
        }
        fence_barrier_init();
        s_abort = 0;
    }
    const int nwu = (nb + 31) >> 5;
    // the group's bitset rows [G][nw] and the table row borrow the stage buffers
    // (no TMA in flight yet); the table row goes there whole when it fits and the
    // table is 16-byte aligned, else its entries are read from global memory
    uint32_t* wbits = reinterpret_cast<uint32_t*>(stages);
    int32_t* trow_area = reinterpret_cast<int32_t*>(wbits + G4 * a.nw);
    const bool trow_smem = ((reinterpret_cast<uintptr_t>(c.table) & 15) == 0) &&
                           (size_t)(G4 * a.nw + c.mbp + 4) * 4 <= (size_t)STAGES * Cfg::STAGE_BYTES;
    __shared__ int32_t* s_trow;
    uint32_t* qraw = reinterpret_cast<uint32_t*>(qs);       // [G][D] bf16 pairs
    stage_query_vec(static_cast<const __nv_bfloat16*>(a.q), a.aw, c.m, c.table, c.mbp, c.hq, c.hkv,
                    G, D, b, h, qraw, aw, ml, (nb > 0 && trow_smem) ? trow_area : nullptr,
                    &s_trow, tid, blockDim.x);
    __syncthreads();
    const int32_t* trow = (nb > 0 && trow_smem) ? s_trow : c.table + (int64_t)b * c.mbp;
    // consumers' B fragments, still before the wait: column n = lane/4; rows
    // k = 2*(lane%4) (+1, +8, +9) of each 16-dim step
    uint32_t qf[D / 16][2], wf[D / 16][2];
    if (warp < NCW) {
        const int n = lane >> 2;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int kb = kk * 16 + 2 * (lane & 3);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int i = kb + 8 * half;
                qf[kk][half] = (n < G) ? qraw[(n * D + i) >> 1] : 0u;
                uint32_t wv = 0u;
                const int g = n & 3;
                if (g < G) {
                    const float x0 = aw[i * 4 + g], x1 = aw[(i + 1) * 4 + g];
                    const uint32_t hi = pack_bf16(x0, x1);
                    wv = (n < 4) ? hi : pack_bf16(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
                }
                wf[kk][half] = wv;
            }
        }
    }
    pdl_wait();
    if (tid == 0) stamp_first(a.stamps, kStampDecode);
    // the group's selections (one round of loads by every thread), then every
    // thread builds its words' part of this CTA's share of their union
    if (nb > 0) {
        stage_bits_vec(a.bits, a.nw, c.hq, G, b, h, wbits, tid, blockDim.x);
        __syncthreads();
        const int n = union_share_cta<Cfg::THREADS>(trow, c.num_phys, G, wbits, a.nw, nwu, nb,
                                                    split, nsplit, a.max_per, blk, phys, hm,
                                                    a.status, s_wsum);
        if (tid == 0) s_n[0] = n;
    } else if (tid == 0) {
        s_n[0] = 0;
    }
    __syncthreads();
    const int nblk = s_n[0];

    if (nb == 0) {
        for (int e = tid; e < G * REC; e += blockDim.x) {
            const int g = e / REC, f = e % REC;
            a.part[(rec_base + g) * REC + f] = (f == 0) ? -SPLA_INF : 0.f;
        }
        if (tid == 0) stamp_last(a.stamps, kStampDecode);
        return;
    }

    // per-lane consumer state: columns c0, c1 of the 16x8 C fragments
    float m_run[2] = {-SPLA_INF, -SPLA_INF}, l_run[2] = {0.f, 0.f}, dt_run[2] = {0.f, 0.f};
    float acc[D / 16][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    const int c0 = 2 * (lane & 3), c1 = c0 + 1;

    if (warp == NCW) {
        // ---------------- producer: TMA ring over 64-token units
        if (lane == 0) {
            fence_proxy_async();   // order this CTA's generic shared-memory writes before TMA
            int u = 0;
            for (int it = 0; it < nblk && !s_abort; ++it) {
                for (int half = 0; half < UPB; ++half) {
                    if (blk[it] * BS + half * 64 >= L) break;
                    const int st = u % STAGES;
                    if (u >= STAGES && !mbar_wait_bounded(&empty[st], ((u / STAGES) - 1) & 1)) {
                        set_status(a.status, SPLA_DEV_TIMEOUT);
                        atomicExch(&s_abort, 1);
                        break;
                    }
                    unsigned char* kst = stages + st * Cfg::STAGE_BYTES;
                    unsigned char* vst = kst + Cfg::TILE_BYTES;
                    mbar_arrive_expect_tx(&full[st], Cfg::STAGE_BYTES);
                    const int row = (phys[it] * c.hkv + h) * BS + half * 64;
#pragma unroll
                    for (int bx = 0; bx < Cfg::BOXES; ++bx) {
                        tma_load_2d(kst + bx * Cfg::BOX_BYTES, &tmK, &full[st], bx * 64, row);
                        tma_load_2d(vst + bx * Cfg::BOX_BYTES, &tmV, &full[st], bx * 64, row);
                    }
                    ++u;
                }
            }
        }
    } else {
        // ---------------- consumers
        const bool lo_half = (lane & 3) < 2;
        const int qm = lane >> 3, rr = lane & 7;
        const int t0 = warp * 16;                       // this warp's slab of every unit
        int u = 0;
        bool stop = false;
        for (int it = 0; it < nblk && !stop; ++it) {
            const int jblk = blk[it];
            const uint32_t hmask = hm[it];
            for (int half = 0; half < UPB; ++half) {
                const int tb = jblk * BS + half * 64;
                if (tb >= L) break;
                const int nvalid = min(64, L - tb);
                const int st = u % STAGES;
                if (!mbar_wait_bounded(&full[st], (u / STAGES) & 1)) {
                    set_status(a.status, SPLA_DEV_TIMEOUT);
                    atomicExch(&s_abort, 1);
                    stop = true;
                    break;
                }
                const unsigned char* kst = stages + st * Cfg::STAGE_BYTES;
                unsigned char* vst = const_cast<unsigned char*>(kst) + Cfg::TILE_BYTES;
                const uint32_t kbase = smem_u32(kst), vbase = smem_u32(vst);
                if (hmask && t0 < nvalid) {
                    if (t0 + 16 > nvalid) {
                        // rows past the sequence end: zero V so that p = 0 rows add nothing
                        for (int e = lane; e < 16 * (D / 8); e += 32) {
                            const int r = t0 + e / (D / 8), ch = e % (D / 8);
                            if (r >= nvalid)
                                *reinterpret_cast<uint4*>(vst + (ch >> 3) * Cfg::BOX_BYTES +
                                                          swz128(r, ch & 7)) = make_uint4(0, 0, 0, 0);
                        }
                        fence_proxy_async();
                        __syncwarp();
                    }
                    // two logit accumulators (even/odd 16-dim steps) halve the MMA chain
                    float cl[4] = {0.f, 0.f, 0.f, 0.f}, cl2[4] = {0.f, 0.f, 0.f, 0.f};
                    float cw1[4] = {0.f, 0.f, 0.f, 0.f}, cw2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const int t = t0 + rr + ((qm & 1) << 3);
                        const int ch = ((kk & 3) << 1) + (qm >> 1);
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4(kbase + (kk >> 2) * Cfg::BOX_BYTES + swz128(t, ch), a0, a1, a2, a3);
                        mma_bf16((kk & 1) ? cl2 : cl, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
                        const int kb = kk * 16 + 2 * (lane & 3);
                        const float2 mA = *reinterpret_cast<const float2*>(ml + kb);
                        const float2 mB = *reinterpret_cast<const float2*>(ml + kb + 8);
                        uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
                        // phi = exp(k - m) of a bf16 pair, split into bf16 hi + lo
                        auto phi = [&](uint32_t kr, float m0, float m1, uint32_t& hi, uint32_t& lo) {
                            const float x0 = ex2(fmaf(bf16_lo(kr), SPLA_LOG2E, -m0));
                            const float x1 = ex2(fmaf(bf16_hi(kr), SPLA_LOG2E, -m1));
                            hi = pack_bf16(x0, x1);
                            lo = pack_bf16(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
                        };
                        phi(a0, mA.x, mA.y, h0, l0);
                        phi(a1, mA.x, mA.y, h1, l1);
                        phi(a2, mB.x, mB.y, h2, l2);
                        phi(a3, mB.x, mB.y, h3, l3);
                        mma_bf16(cw1, h0, h1, h2, h3, wf[kk][0], wf[kk][1]);
                        mma_bf16(cw2, l0, l1, l2, l3, wf[kk][0], wf[kk][1]);
                    }
                    // W = hi-part columns + lo-part columns (cols g and g+4)
                    float x[4], y[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) cl[r] += cl2[r];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        x[r] = cw1[r] + cw2[r];
                        y[r] = __shfl_down_sync(0xffffffffu, x[r], 2);
                    }
                    const int tr0 = t0 + (lane >> 2), tr1 = tr0 + 8;
                    const bool hc0 = lo_half && c0 < G && ((hmask >> c0) & 1u);
                    const bool hc1 = lo_half && c1 < G && ((hmask >> c1) & 1u);
                    const bool v00 = hc0 && tr0 < nvalid, v01 = hc1 && tr0 < nvalid;
                    const bool v10 = hc0 && tr1 < nvalid, v11 = hc1 && tr1 < nvalid;
                    const float s00 = v00 ? cl[0] * a.sl2 : -SPLA_INF;
                    const float s01 = v01 ? cl[1] * a.sl2 : -SPLA_INF;
                    const float s10 = v10 ? cl[2] * a.sl2 : -SPLA_INF;
                    const float s11 = v11 ? cl[3] * a.sl2 : -SPLA_INF;
                    const float w00 = v00 ? x[0] + y[0] : 0.f, w01 = v01 ? x[1] + y[1] : 0.f;
                    const float w10 = v10 ? x[2] + y[2] : 0.f, w11 = v11 ? x[3] + y[3] : 0.f;
                    float mx0 = fmaxf(s00, s10), mx1 = fmaxf(s01, s11);
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) {
                        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
                        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
                    }
                    const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
                    const float f0 = (mn0 == -SPLA_INF) ? 1.f : ex2(m_run[0] - mn0);
                    const float f1 = (mn1 == -SPLA_INF) ? 1.f : ex2(m_run[1] - mn1);
                    const float p00 = v00 ? ex2(s00 - mn0) : 0.f, p10 = v10 ? ex2(s10 - mn0) : 0.f;
                    const float p01 = v01 ? ex2(s01 - mn1) : 0.f, p11 = v11 ? ex2(s11 - mn1) : 0.f;
                    l_run[0] = l_run[0] * f0 + p00 + p10;
                    l_run[1] = l_run[1] * f1 + p01 + p11;
                    m_run[0] = mn0;
                    m_run[1] = mn1;
                    dt_run[0] += w00 + w10;
                    dt_run[1] += w01 + w11;
                    const float g0 = lo_half ? f0 : 1.f, g1 = lo_half ? f1 : 1.f;
                    // the running maxima rarely move once the first tiles are in
                    if (!__all_sync(0xffffffffu, g0 == 1.f && g1 == 1.f)) {
#pragma unroll
                        for (int mt = 0; mt < D / 16; ++mt) {
                            acc[mt][0] *= g0;
                            acc[mt][1] *= g1;
                            acc[mt][2] *= g0;
                            acc[mt][3] *= g1;
                        }
                    }
                    // [P | W] as a 16 x 8 matrix in C layout: lanes with cols 4..7 take W from lane-2
                    const float wv[4] = {w00, w01, w10, w11};
                    const float pv[4] = {p00, p01, p10, p11};
                    float pw[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const float up = __shfl_up_sync(0xffffffffu, wv[r], 2);
                        pw[r] = lo_half ? pv[r] : up;
                    }
                    const uint32_t hA = pack_bf16(pw[0], pw[1]), hB = pack_bf16(pw[2], pw[3]);
                    const uint32_t lA = pack_bf16(pw[0] - bf16_lo(hA), pw[1] - bf16_hi(hA));
                    const uint32_t lB = pack_bf16(pw[2] - bf16_lo(hB), pw[3] - bf16_hi(hB));
                    const uint32_t bh0 = movmatrix_t(hA), bh1 = movmatrix_t(hB);
                    const uint32_t bl0 = movmatrix_t(lA), bl1 = movmatrix_t(lB);
#pragma unroll
                    for (int mt = 0; mt < D / 16; ++mt) {
                        const int t = t0 + rr + ((qm >> 1) << 3);
                        const int ch = ((mt & 3) << 1) + (qm & 1);
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4_t(vbase + (mt >> 2) * Cfg::BOX_BYTES + swz128(t, ch), a0, a1, a2, a3);
                        mma_bf16(acc[mt], a0, a1, a2, a3, bh0, bh1);
                        mma_bf16(acc[mt], a0, a1, a2, a3, bl0, bl1);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
                ++u;
            }
        }
        // reduce the lane partials of l and D~ over the 8 lanes of each column
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                l_run[e] += __shfl_xor_sync(0xffffffffu, l_run[e], o);
                dt_run[e] += __shfl_xor_sync(0xffffffffu, dt_run[e], o);
            }
    }
    // every consumer is done with the stage buffers once all threads pass here
    __syncthreads();
    float* mw = reinterpret_cast<float*>(stages);           // [NCW][4]
    float* lw = mw + NCW * 4;
    float* dw = lw + NCW * 4;
    // per-warp partial rows [NCW][4][D + 4]; the N~ rows start 16 floats further so
    // that the four lanes writing one column hit four different bank groups
    constexpr int RP = D + 4;
    float* ap = dw + NCW * 4;                               // 16-byte aligned (48 floats in)
    float* an = ap + NCW * 4 * RP + 16;
    if (warp < NCW) {
        if (lane < 2) {
            mw[warp * 4 + c0] = m_run[0];
            mw[warp * 4 + c1] = m_run[1];
            lw[warp * 4 + c0] = l_run[0];
            lw[warp * 4 + c1] = l_run[1];
            dw[warp * 4 + c0] = dt_run[0];
            dw[warp * 4 + c1] = dt_run[1];
        }
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int j = mt * 16 + (lane >> 2) + ((r >> 1) << 3);
                const int col = 2 * (lane & 3) + (r & 1);
                float* dst = (col < 4) ? ap + (warp * 4 + col) * RP : an + (warp * 4 + col - 4) * RP;
                dst[j] = acc[mt][r];
            }
    }
    __syncthreads();
    // merge the consumer warps and write the partial records, four columns a thread
    for (int e = tid; e < G * (D / 4); e += blockDim.x) {
        const int g = e / (D / 4), j = 4 * (e % (D / 4));
        float M = -SPLA_INF;
        for (int w = 0; w < NCW; ++w) M = fmaxf(M, mw[w * 4 + g]);
        float l = 0.f, dt = 0.f;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f), nt = o;
#pragma unroll
        for (int w = 0; w < NCW; ++w) {
            const float f = (M == -SPLA_INF) ? 0.f : ex2(mw[w * 4 + g] - M);
            l += lw[w * 4 + g] * f;
            dt += dw[w * 4 + g];
            const float4 pa = *reinterpret_cast<const float4*>(ap + (w * 4 + g) * RP + j);
            const float4 pn = *reinterpret_cast<const float4*>(an + (w * 4 + g) * RP + j);
            o.x += pa.x * f; o.y += pa.y * f; o.z += pa.z * f; o.w += pa.w * f;
            nt.x += pn.x; nt.y += pn.y; nt.z += pn.z; nt.w += pn.w;
        }
        float* rec = a.part + (rec_base + g) * REC;
        *reinterpret_cast<float4*>(rec + 4 + j) = o;
        *reinterpret_cast<float4*>(rec + 4 + D + j) = nt;
        if (j == 0) *reinterpret_cast<float4*>(rec) = make_float4(M, l, dt, 0.f);
    }
    if (tid == 0) stamp_last(a.stamps, kStampDecode);
}

// ------------------------------------------------------------------ fp32 SIMT kernel
// One CTA of 256 threads per (split, group). Tiles are staged through shared
// memory as fp32; every product and sum is an fp32 FMA.
template <typename T>
__global__ void __launch_bounds__(256) decode_simt_kernel(const __grid_constant__ CacheView c,
                                                          const __grid_constant__ DecodeArgs a) {
    extern __shared__ __align__(16) unsigned char smem_simt[];
    const int d = c.d, BS = c.bs, G = c.group;
    float* Ks = reinterpret_cast<float*>(smem_simt);       // [BS][d]
    float* Vs = Ks + BS * d;                                // [BS][d]
    float* Ls = Vs + BS * d;                                // [4][BS] logits, then p
    float* Ws = Ls + 4 * BS;                                // [4][BS] phi weights
    float* qs = Ws + 4 * BS;                                // [4][d]
    float* aw = qs + 4 * d;                                 // [4][d]
    float* ml = aw + 4 * d;                                 // [d]
    float* cg = ml + d;                                     // [4]
    float* fsc = cg + 4;                                    // [4] per-head rescale of this tile
    int32_t* blk = reinterpret_cast<int32_t*>(fsc + 4);
    int32_t* phys = blk + a.max_per;
    uint32_t* hm = reinterpret_cast<uint32_t*>(phys + a.max_per);
    __shared__ int s_n[2];
    __shared__ float s_m[4], s_l[4], s_dt[4];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y / c.hkv, h = blockIdx.y % c.hkv, split = blockIdx.x;
    const int nsplit = a.nsplit;
    pdl_trigger();
    int32_t L = c.lens[b];
    if (L < 0 || L > c.mbp * c.bs) L = max(0, min(L, c.mbp * c.bs));
    const int nb = (L + BS - 1) / BS;
    const int64_t rec_base = (((int64_t)b * c.hkv + h) * nsplit + split) * G;
    const int REC = rec_floats(d);
    if (nb == 0) {
        for (int e = tid; e < G * REC; e += blockDim.x) {
            const int g = e / REC, f = e % REC;
            a.part[(rec_base + g) * REC + f] = (f == 0) ? -SPLA_INF : 0.f;
        }
        return;
    }
    // bitset words and counts borrow the K and V tiles
    const int nwu = (nb + 31) >> 5;
    uint32_t* wbits = reinterpret_cast<uint32_t*>(Ks);
    stage_query(a.q, a.aw, c.m, c.table, c.mbp, c.hq, c.hkv, G, d, sizeof(T) == 2, b, h, qs, ml,
                aw, nullptr, tid, blockDim.x);
    pdl_wait();
    if (tid == 0) stamp_first(a.stamps, kStampDecode);
    stage_bits(a.bits, a.nw, c.hq, G, b, h, nwu, wbits, tid, blockDim.x);
    __syncthreads();
    const int nblk = union_share(c.table + (int64_t)b * c.mbp, c.num_phys, G, wbits, nwu, nb,
                                 split, nsplit, a.max_per, reinterpret_cast<int*>(wbits + G * nwu),
                                 blk, phys, hm, s_n, a.status, tid, blockDim.x);
    if (tid < 4) { s_m[tid] = -SPLA_INF; s_l[tid] = 0.f; s_dt[tid] = 0.f; }
    __syncthreads();
    // accumulators: thread owns (g, j) pairs e = tid + 256*u
    constexpr int PU = 2;                                   // G*d <= 512
    float acc[PU] = {0.f, 0.f}, ntl[PU] = {0.f, 0.f};
    for (int it = 0; it < nblk; ++it) {
        const int jblk = blk[it];
        const int nvalid = min(BS, L - jblk * BS);
        const uint32_t hmask = hm[it];
        __syncthreads();
        const T* kp = (const T*)c.k_pool + ((int64_t)phys[it] * c.hkv + h) * BS * d;
        const T* vp = (const T*)c.v_pool + ((int64_t)phys[it] * c.hkv + h) * BS * d;
        for (int e = tid; e < BS * d; e += blockDim.x) {
            const bool ok = (e / d) < nvalid;
            Ks[e] = ok ? to_f(kp[e]) : 0.f;
            Vs[e] = ok ? to_f(vp[e]) : 0.f;
        }
        __syncthreads();
        // logits and phi weights per (g, t); dimension order rotated by t (no bank conflicts)
        for (int e = tid; e < 4 * BS; e += blockDim.x) {
            const int g = e / BS, t = e % BS;
            float lg = -SPLA_INF, w = 0.f;
            if (g < G && t < nvalid && ((hmask >> g) & 1u)) {
                float sacc = 0.f, wacc = 0.f;
                for (int u = 0; u < d; ++u) {
                    const int i = (u + t) & (d - 1);
                    const float kv = Ks[t * d + i];
                    sacc = fmaf(qs[g * d + i], kv, sacc);
                    wacc = fmaf(aw[g * d + i], ex2(fmaf(kv, SPLA_LOG2E, -ml[i])), wacc);
                }
                lg = sacc * a.sl2;
                w = wacc;
            }
            Ls[e] = lg;
            Ws[e] = w;
        }
        __syncthreads();
        // online softmax, one warp per head
        if (warp < G) {
            float mx = -SPLA_INF;
            for (int t = lane; t < BS; t += 32) mx = fmaxf(mx, Ls[warp * BS + t]);
            mx = warp_max(mx);
            const float mo = s_m[warp];
            const float mn = fmaxf(mo, mx);
            const float f = (mn == -SPLA_INF) ? 1.f : ex2(mo - mn);
            float ls = 0.f, ds = 0.f;
            for (int t = lane; t < BS; t += 32) {
                const float lv = Ls[warp * BS + t];
                const float p = (lv == -SPLA_INF) ? 0.f : ex2(lv - mn);
                Ls[warp * BS + t] = p;
                ls += p;
                ds += Ws[warp * BS + t];
            }
            ls = warp_sum(ls);
            ds = warp_sum(ds);
            if (lane == 0) {
                s_m[warp] = mn;
                s_l[warp] = s_l[warp] * f + ls;
                s_dt[warp] += ds;
                fsc[warp] = f;
            }
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < PU; ++u) {
            const int e = tid + 256 * u;
            if (e < G * d) {
                const int g = e / d, j = e % d;
                float av = acc[u] * fsc[g], n = ntl[u];
                for (int t = 0; t < nvalid; ++t) {
                    const float vv = Vs[t * d + j];
                    av = fmaf(Ls[g * BS + t], vv, av);
                    n = fmaf(Ws[g * BS + t], vv, n);
                }
                acc[u] = av;
                ntl[u] = n;
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < PU; ++u) {
        const int e = tid + 256 * u;
        if (e < G * d) {
            const int g = e / d, j = e % d;
            float* rec = a.part + (rec_base + g) * REC;
            rec[4 + j] = acc[u];
            rec[4 + d + j] = ntl[u];
            if (j == 0) {
                rec[0] = s_m[g];
                rec[1] = s_l[g];
                rec[2] = s_dt[g];
                rec[3] = 0.f;
            }
        }
    }
    if (tid == 0) stamp_last(a.stamps, kStampDecode);
}

// ------------------------------------------------------------------ host launchers
template <int D, int UPB, int STAGES>
static size_t mma_smem_bytes(int max_per) {
    using Cfg = MmaCfg<D, UPB, STAGES>;
    return 1024 + (size_t)STAGES * Cfg::STAGE_BYTES + 2 * STAGES * sizeof(uint64_t) +
           3 * (size_t)max_per * 4 + 16 + (size_t)(4 * D * 2 + D + 4) * 4 + 64;
}

template <int D, int UPB, int STAGES>
static cudaError_t launch_mma_t(const CacheView& c, const CUtensorMap& tk, const CUtensorMap& tv,
                                const DecodeArgs& a, cudaStream_t s) {
    using Cfg = MmaCfg<D, UPB, STAGES>;
    const size_t smem = mma_smem_bytes<D, UPB, STAGES>(a.max_per);
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel<D, UPB, STAGES>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // all of the unified L1/shared array as shared memory: three CTAs per SM need it
    e = cudaFuncSetAttribute(decode_mma_kernel<D, UPB, STAGES>,
                             cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    dim3 grid(a.nsplit, c.batch * c.hkv);
    return launch_pdl(decode_mma_kernel<D, UPB, STAGES>, grid, dim3(Cfg::THREADS), smem, s, c, tk,
                      tv, a);
}

// The merge area reuses the stage ring; it must fit.
static_assert(2 * MmaCfg<128, 1, 2>::STAGE_BYTES >= (2 * 4 * 4 * 132 + 16 + 48) * 4, "merge area");
static_assert(4 * MmaCfg<64, 1, 4>::STAGE_BYTES >= (2 * 4 * 4 * 68 + 16 + 48) * 4, "merge area");

size_t mma_smem_for(int d, int bs, int max_per) {
    if (d == 128) return bs == 64 ? mma_smem_bytes<128, 1, 2>(max_per) : mma_smem_bytes<128, 2, 2>(max_per);
    return bs == 64 ? mma_smem_bytes<64, 1, 4>(max_per) : mma_smem_bytes<64, 2, 4>(max_per);
}

cudaError_t launch_decode_mma(const CacheView& c, const CUtensorMap& tk, const CUtensorMap& tv,
                              const DecodeArgs& a, cudaStream_t s) {
    if (c.d == 128 && c.bs == 64) return launch_mma_t<128, 1, 2>(c, tk, tv, a, s);
    if (c.d == 128 && c.bs == 128) return launch_mma_t<128, 2, 2>(c, tk, tv, a, s);
    if (c.d == 64 && c.bs == 64) return launch_mma_t<64, 1, 4>(c, tk, tv, a, s);
    return launch_mma_t<64, 2, 4>(c, tk, tv, a, s);
}

size_t simt_smem_for(int d, int bs, int max_per) {
    const size_t tiles = (size_t)(2 * bs * d + 8 * bs + 4 * d * 2 + d + 8) * 4;
    return tiles + 3 * (size_t)max_per * 4 + 64;
}

cudaError_t launch_decode_simt(const CacheView& c, int dtype, const DecodeArgs& a, cudaStream_t s) {
    const size_t smem = simt_smem_for(c.d, c.bs, a.max_per);
    dim3 grid(a.nsplit, c.batch * c.hkv);
    cudaError_t e;
    if (dtype == SPLA_BF16) {
        e = cudaFuncSetAttribute(decode_simt_kernel<__nv_bfloat16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(decode_simt_kernel<__nv_bfloat16>, grid, dim3(256), smem, s, c, a);
    } else {
        e = cudaFuncSetAttribute(decode_simt_kernel<float>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(decode_simt_kernel<float>, grid, dim3(256), smem, s, c, a);
    }
}

cudaError_t launch_combine(const CacheView& c, int dtype, const DecodeArgs& a, cudaStream_t s) {
    const size_t smem = (size_t)5 * a.nsplit * sizeof(float);
    const dim3 grid(c.batch * c.hq), block(kCombThreads);
    if (c.d == 128)
        return dtype == SPLA_BF16
            ? launch_pdl(combine_kernel<128, __nv_bfloat16>, grid, block, smem, s, c, a)
            : launch_pdl(combine_kernel<128, float>, grid, block, smem, s, c, a);
    return dtype == SPLA_BF16
        ? launch_pdl(combine_kernel<64, __nv_bfloat16>, grid, block, smem, s, c, a)
        : launch_pdl(combine_kernel<64, float>, grid, block, smem, s, c, a);
}

}  // namespace spla
