// a1 + a2 -- block scoring and top-k selection (SPLA technical summary,
// gist.science, section 2.1: the block relevance is the integrated attention
// mass of its tokens, approximated around the block mean by
// exp(q.kbar)(1 + 1/2 q^T diag(sigma^2) q); the blocks with the largest
// estimates are attended exactly).
//
// score_kernel  grid (chunks, batch*Hkv), 4 warps. Streams each block's
//               statistics (1 KiB at d=128) once per KV head and scores it for
//               all G query heads of the group. Lane l of a warp owns block
//               jb + l: it walks the block's mean and variance in 16-byte
//               loads and accumulates the G x 2 dot products in fp64 against
//               {q', q'^2} broadcast from shared memory (no cross-lane work);
//               the log-domain score is finished per lane.
// select_kernel grid (batch*Hq), 512 threads. Exact top-k by key-space
//               bucketing: 2048 linear buckets over the live key range, the
//               bucket holding the k-th key is refined until few candidates
//               remain, which are ranked pairwise (ties -> lower block index).
//               Writes a per-head selection bitset (warp ballots over 32
//               consecutive blocks), the sorted block list and its length, and
//               clears the group's completion counter for the decode kernel.
#include "common.cuh"

namespace spla {

constexpr int kScoreThreads = 128;     // 4 warps; a warp scores 32 blocks at once

template <int D, typename T>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(CacheView c, const T* __restrict__ q,
                                                              double scale, int first_order,
                                                              float* __restrict__ scores,
                                                              int chunk, int32_t* status) {
    __shared__ double2 qsm[4][D];                  // {q', q'^2} per head and dimension
    const int b = blockIdx.y / c.hkv, h = blockIdx.y % c.hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t L = c.lens[b];
    if (L < 0 || L > c.mbp * c.bs) {
        if (blockIdx.x == 0 && threadIdx.x == 0 && h == 0) set_status(status, SPLA_DEV_CAPACITY);
        L = max(0, min(L, c.mbp * c.bs));
    }
    const int nb = (L + c.bs - 1) / c.bs;
    const int j0 = blockIdx.x * chunk;
    if (j0 >= nb) return;
    const int j1 = min(nb, j0 + chunk);
    const int G = c.group;
    for (int e = threadIdx.x; e < 4 * D; e += blockDim.x) {
        const int g = e / D, i = e % D;
        double v = 0.0;
        if (g < G) v = (double)to_f(q[((int64_t)b * c.hq + h * G + g) * D + i]) * scale;
        qsm[g][i] = make_double2(v, v * v);
    }
    __syncthreads();
    const int nwarps = blockDim.x >> 5;
    for (int jb = j0 + warp * 32; jb < j1; jb += 32 * nwarps) {
        const int j = jb + lane;
        bool ok = false;
        const float* st = c.stats;
        if (j < j1) {
            const int32_t phys = c.table[(int64_t)b * c.mbp + j];
            ok = phys >= 0 && phys < c.num_phys;
            if (ok) st = c.stats + ((int64_t)phys * c.hkv + h) * 2 * D;
            else set_status(status, SPLA_DEV_BAD_BLOCK_TABLE);
        }
        double s1[4] = {0.0, 0.0, 0.0, 0.0}, s2[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
        for (int i0 = 0; i0 < D; i0 += 4) {
            float4 m4 = make_float4(0.f, 0.f, 0.f, 0.f), v4 = m4;
            if (ok) {
                m4 = __ldg(reinterpret_cast<const float4*>(st + i0));
                v4 = __ldg(reinterpret_cast<const float4*>(st + D + i0));
            }
            const float mu[4] = {m4.x, m4.y, m4.z, m4.w}, va[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const double dm = (double)mu[u], dv = (double)va[u];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    if (g < G) {
                        const double2 qq = qsm[g][i0 + u];
                        s1[g] = fma(qq.x, dm, s1[g]);
                        s2[g] = fma(qq.y, dv, s2[g]);
                    }
                }
            }
        }
        if (j < j1) {
            const int nj = min(c.bs, L - j * c.bs);
            const double ln = log((double)nj);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                if (g < G) {
                    double sc = ln + s1[g];
                    if (!first_order) sc += log1p(0.5 * s2[g]);
                    scores[((int64_t)b * c.hq + h * G + g) * c.mbp + j] = ok ? (float)sc : -SPLA_INF;
                }
            }
        }
    }
}

// ------------------------------------------------------------------ selection
constexpr int kSelThreads = 512;
constexpr int kBins = 2048;
constexpr int kCandCap = 256;

__device__ int block_excl_scan(int v, int* tmp, int* total) {
    // tmp: >= 33 ints of shared memory
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int t = lane < nw ? tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        if (lane < nw) tmp[lane] = t;             // inclusive warp totals
        if (lane == 31) tmp[32] = t;
    }
    __syncthreads();
    const int before = (warp > 0 ? tmp[warp - 1] : 0) + x - v;
    if (total) *total = tmp[32];
    __syncthreads();
    return before;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(CacheView c, int top_k, int n_sink,
                                                             int n_local, const float* scores,
                                                             uint32_t* bits, int nw,
                                                             int32_t* nsel, int32_t* sel_idx,
                                                             int kcap, int32_t* counters) {
    extern __shared__ __align__(16) unsigned char smem_sel[];
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem_sel);        // [mbp padded]
    __shared__ int hist[kBins];
    __shared__ int wpre[SPLA_MAX_BLOCKS_PER_SEQ / 32];             // per-word counts, then prefixes
    __shared__ uint32_t cand_key[kCandCap];
    __shared__ int cand_idx[kCandCap];
    __shared__ int tmp[40];
    __shared__ unsigned long long s_lo, s_hi;
    __shared__ int s_krem, s_cnt, s_done, s_mode, s_ncand, s_total;
    __shared__ uint32_t s_min, s_max;

    const int b = blockIdx.x / c.hq, hq = blockIdx.x % c.hq;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0 && hq % c.group == 0) counters[(int64_t)b * c.hkv + hq / c.group] = 0;
    int32_t L = c.lens[b];
    L = max(0, min(L, c.mbp * c.bs));
    const int nb = (L + c.bs - 1) / c.bs;
    const float* sc = scores + ((int64_t)b * c.hq + hq) * c.mbp;
    // block j belongs to thread j % kSelThreads; rounds of kSelThreads consecutive blocks
    const int rounds = (nb + kSelThreads - 1) / kSelThreads;

    const int fs = min(n_sink, nb), fl0 = max(0, nb - n_local);
    auto forced = [&](int j) { return j < fs || j >= fl0; };
    int nforced = fs + (nb - fl0);
    if (fl0 < fs) nforced = nb;                     // overlapping ranges
    const int ncand = nb - nforced;
    const bool take_all = ncand <= top_k;

    if (tid == 0) { s_min = 0xffffffffu; s_max = 0u; }
    __syncthreads();
    uint32_t lmin = 0xffffffffu, lmax = 0u;
    for (int j = tid; j < nb; j += kSelThreads) {
        const uint32_t k = forced(j) ? 0u : ordered_key(sc[j]);
        keys[j] = k;
        if (k) { lmin = min(lmin, k); lmax = max(lmax, k); }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        lmin = min(lmin, __shfl_xor_sync(0xffffffffu, lmin, o));
        lmax = max(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    }
    if (lane == 0 && !take_all) {
        atomicMin(&s_min, lmin);
        atomicMax(&s_max, lmax);
    }
    __syncthreads();

    if (!take_all) {
        if (tid == 0) {
            s_lo = s_min;
            s_hi = (unsigned long long)s_max + 1ull;
            s_krem = top_k;
            s_done = 0;
            s_mode = 0;
        }
        __syncthreads();
        for (int pass = 0; pass < 8 && !s_done; ++pass) {
            const unsigned long long lo = s_lo, hi = s_hi;
            int shift = 0;
            while (((hi - lo - 1ull) >> shift) >= (unsigned long long)kBins) ++shift;
            const int nbins = (int)((hi - lo - 1ull) >> shift) + 1;
            for (int i = tid; i < nbins; i += kSelThreads) hist[i] = 0;
            __syncthreads();
            for (int j = tid; j < nb; j += kSelThreads) {
                const unsigned long long k = keys[j];
                if (k >= lo && k < hi) atomicAdd(&hist[(int)((k - lo) >> shift)], 1);
            }
            __syncthreads();
            // suffix scan from the top bucket; thread t covers reversed buckets [4t, 4t+4)
            int local[4], lsum = 0;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = 4 * tid + u;
                local[u] = (r < nbins) ? hist[nbins - 1 - r] : 0;
                lsum += local[u];
            }
            const int before = block_excl_scan(lsum, tmp, nullptr);
            const int krem = s_krem;
            if (before < krem && before + lsum >= krem) {
                int acc = before;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (acc < krem && acc + local[u] >= krem) {
                        const int bstar = nbins - 1 - (4 * tid + u);
                        const unsigned long long nlo = lo + ((unsigned long long)bstar << shift);
                        unsigned long long nhi = lo + ((unsigned long long)(bstar + 1) << shift);
                        if (nhi > hi) nhi = hi;
                        s_lo = nlo;
                        s_hi = nhi;
                        s_krem = krem - acc;        // still to take from [nlo, nhi)
                        s_cnt = local[u];
                    }
                    acc += local[u];
                }
            }
            __syncthreads();
            if (tid == 0) {
                if (s_cnt == s_krem) { s_mode = 1; s_done = 1; }            // the whole bucket
                else if (s_cnt <= kCandCap) { s_mode = 2; s_done = 1; }     // rank candidates
                else if (s_hi - s_lo == 1ull) { s_mode = 3; s_done = 1; }   // all equal: by index
                else s_mode = 0;
                s_ncand = 0;
            }
            __syncthreads();
        }
        const unsigned long long lo = s_lo, hi = s_hi;
        const int krem = s_krem;
        if (s_mode == 1) {
            // every key in [lo, hi) is selected: lift them above the final threshold
            for (int j = tid; j < nb; j += kSelThreads)
                if (keys[j] >= lo && keys[j] < hi) keys[j] = 0xffffffffu;
        } else if (s_mode == 2) {
            for (int r = 0; r < rounds; ++r) {
                const int j = r * kSelThreads + tid;
                const bool in = j < nb && keys[j] >= lo && keys[j] < hi;
                const uint32_t m = __ballot_sync(0xffffffffu, in);
                int base = 0;
                if (lane == 0 && m) base = atomicAdd(&s_ncand, __popc(m));
                base = __shfl_sync(0xffffffffu, base, 0);
                if (in) {
                    const int p = base + __popc(m & ((1u << lane) - 1u));
                    if (p < kCandCap) { cand_key[p] = keys[j]; cand_idx[p] = j; }
                }
            }
            __syncthreads();
            const int nc = min(s_ncand, kCandCap);
            for (int i = tid; i < nc; i += kSelThreads) {
                int rank = 0;
                for (int o = 0; o < nc; ++o)
                    rank += (cand_key[o] > cand_key[i]) ||
                            (cand_key[o] == cand_key[i] && cand_idx[o] < cand_idx[i]);
                if (rank < krem) keys[cand_idx[i]] = 0xffffffffu;
            }
        } else {
            // equal keys: the krem lowest indices among keys == lo, in index order
            int taken = 0;
            for (int r = 0; r < rounds; ++r) {
                const int j = r * kSelThreads + tid;
                const bool eq = j < nb && keys[j] == lo;
                int tot;
                const int rank = taken + block_excl_scan(eq ? 1 : 0, tmp, &tot);
                if (eq && rank < krem) keys[j] = 0xffffffffu;
                taken += tot;
            }
        }
        __syncthreads();
    }

    // flags -> bitset words (one ballot per 32 consecutive blocks), then list positions
    const unsigned long long thr = take_all ? 0ull : s_hi;
    uint32_t* hb = bits + ((int64_t)b * c.hq + hq) * nw;
    const int nwu = (nb + 31) >> 5;
    for (int r = 0; r < rounds; ++r) {
        const int j = r * kSelThreads + tid;
        const bool sel = j < nb && (take_all || forced(j) || (unsigned long long)keys[j] >= thr);
        const uint32_t word = __ballot_sync(0xffffffffu, sel);
        const int wi = (r * kSelThreads + warp * 32) >> 5;
        if (lane == 0 && wi < nwu) {
            hb[wi] = word;
            wpre[wi] = __popc(word);
        }
    }
    __syncthreads();
    if (warp == 0) {
        // exclusive scan of the per-word counts, 32 consecutive words per lane
        const int wpl = (nwu + 31) >> 5;
        const int w0 = lane * wpl, w1 = min(nwu, w0 + wpl);
        int cnt = 0;
        for (int w = w0; w < w1; ++w) cnt += wpre[w];
        int x = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        int run = x - cnt;
        for (int w = w0; w < w1; ++w) {
            const int v = wpre[w];
            wpre[w] = run;
            run += v;
        }
        if (lane == 31) s_total = x;
    }
    __syncthreads();
    const int total = s_total;
    if (sel_idx) {
        int32_t* out = sel_idx + ((int64_t)b * c.hq + hq) * kcap;
        for (int r = 0; r < rounds; ++r) {
            const int j = r * kSelThreads + tid;
            const int wi = (r * kSelThreads + warp * 32) >> 5;
            if (wi < nwu) {
                const uint32_t word = hb[wi];
                if ((word >> lane) & 1u) {
                    const int pos = wpre[wi] + __popc(word & ((1u << lane) - 1u));
                    if (pos < kcap) out[pos] = j;
                }
            }
        }
        for (int i = total + tid; i < kcap; i += kSelThreads) out[i] = -1;
    }
    if (tid == 0) nsel[(int64_t)b * c.hq + hq] = total;
}

// ------------------------------------------------------------------ host launchers
cudaError_t launch_score(const CacheView& c, int dtype, const void* q, double scale,
                         int first_order, float* scores, int chunk, int32_t* status,
                         cudaStream_t s) {
    dim3 grid((c.mbp + chunk - 1) / chunk, c.batch * c.hkv);
    if (dtype == SPLA_BF16) {
        if (c.d == 128)
            score_kernel<128, __nv_bfloat16><<<grid, kScoreThreads, 0, s>>>(c, (const __nv_bfloat16*)q, scale,
                                                                 first_order, scores, chunk, status);
        else
            score_kernel<64, __nv_bfloat16><<<grid, kScoreThreads, 0, s>>>(c, (const __nv_bfloat16*)q, scale,
                                                                first_order, scores, chunk, status);
    } else {
        if (c.d == 128)
            score_kernel<128, float><<<grid, kScoreThreads, 0, s>>>(c, (const float*)q, scale, first_order,
                                                         scores, chunk, status);
        else
            score_kernel<64, float><<<grid, kScoreThreads, 0, s>>>(c, (const float*)q, scale, first_order,
                                                        scores, chunk, status);
    }
    return cudaGetLastError();
}

cudaError_t launch_select(const CacheView& c, int top_k, int n_sink, int n_local,
                          const float* scores, uint32_t* bits, int nw, int32_t* nsel,
                          int32_t* sel_idx, int kcap, int32_t* counters, cudaStream_t s) {
    const size_t smem = (size_t)((c.mbp + 31) / 32) * 32 * sizeof(uint32_t);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(select_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    select_kernel<<<c.batch * c.hq, kSelThreads, smem, s>>>(c, top_k, n_sink, n_local, scores,
                                                            bits, nw, nsel, sel_idx, kcap,
                                                            counters);
    return cudaGetLastError();
}

}  // namespace spla
