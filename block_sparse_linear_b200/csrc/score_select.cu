// a1 + a2 -- block scoring and top-k selection (SPLA technical summary,
// gist.science, section 2.1: the block relevance is the integrated attention
// mass of its tokens, approximated around the block mean by
// exp(q.kbar)(1 + 1/2 q^T diag(sigma^2) q); the blocks with the largest
// estimates are attended exactly).
//
// score_kernel  grid (chunks, batch*Hkv), 8 warps. Streams each block's
//               statistics (1 KiB at d=128) once per KV head and scores it for
//               all G query heads of the group. A warp takes 8 blocks at a
//               time: lanes split the head dimension, the G x 2 dot products
//               are reduced across lanes in fp64 by a transposing butterfly,
//               and lane 4*b+g finishes block b, head g (one log1p per lane).
// select_kernel grid (batch*Hq), 512 threads. Exact top-k by key-space
//               bucketing: 2048 linear buckets over the live key range, the
//               bucket holding the k-th key is refined until few candidates
//               remain, which are ranked pairwise (ties -> lower block index).
//               Writes a per-head selection bitset, the sorted block list and
//               its length.
#include "common.cuh"

namespace spla {

template <int D, typename T>
__global__ void __launch_bounds__(256) score_kernel(CacheView c, const T* __restrict__ q,
                                                    double scale, int first_order,
                                                    float* __restrict__ scores, int chunk,
                                                    int32_t* status) {
    constexpr int DPL = D / 32;                    // dims per lane: 2 or 4
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

    double qd[4][DPL], q2[4][DPL];
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int u = 0; u < DPL; ++u) {
            double v = 0.0;
            if (g < G) v = (double)to_f(q[((int64_t)b * c.hq + h * G + g) * D + lane * DPL + u]) * scale;
            qd[g][u] = v;
            q2[g][u] = v * v;
        }

    const int nwarps = blockDim.x >> 5;
    for (int jb = j0 + warp * 8; jb < j1; jb += 8 * nwarps) {
        float mu[8][DPL], va[8][DPL];
        bool ok[8];
#pragma unroll
        for (int bb = 0; bb < 8; ++bb) {
            const int j = jb + bb;
            ok[bb] = false;
#pragma unroll
            for (int u = 0; u < DPL; ++u) mu[bb][u] = va[bb][u] = 0.f;
            if (j < j1) {
                const int32_t phys = c.table[(int64_t)b * c.mbp + j];
                if (phys >= 0 && phys < c.num_phys) {
                    ok[bb] = true;
                    const float* st = c.stats + ((int64_t)phys * c.hkv + h) * 2 * D + lane * DPL;
                    if constexpr (DPL == 4) {
                        const float4 m4 = __ldg(reinterpret_cast<const float4*>(st));
                        const float4 v4 = __ldg(reinterpret_cast<const float4*>(st + D));
                        mu[bb][0] = m4.x; mu[bb][1] = m4.y; mu[bb][2] = m4.z; mu[bb][3] = m4.w;
                        va[bb][0] = v4.x; va[bb][1] = v4.y; va[bb][2] = v4.z; va[bb][3] = v4.w;
                    } else {
                        const float2 m2 = __ldg(reinterpret_cast<const float2*>(st));
                        const float2 v2 = __ldg(reinterpret_cast<const float2*>(st + D));
                        mu[bb][0] = m2.x; mu[bb][1] = m2.y;
                        va[bb][0] = v2.x; va[bb][1] = v2.y;
                    }
                } else if (lane == 0) {
                    set_status(status, SPLA_DEV_BAD_BLOCK_TABLE);
                }
            }
        }
        double my1 = 0.0, my2 = 0.0;
#pragma unroll
        for (int bb = 0; bb < 8; ++bb) {
            double v[8];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                double s1 = 0.0, s2 = 0.0;
#pragma unroll
                for (int u = 0; u < DPL; ++u) {
                    s1 = fma(qd[g][u], (double)mu[bb][u], s1);
                    s2 = fma(q2[g][u], (double)va[bb][u], s2);
                }
                v[2 * g] = s1;
                v[2 * g + 1] = s2;
            }
            // transposing butterfly: after it, lanes 4v..4v+3 hold the total of value v
            const bool u16 = lane & 16, u8 = lane & 8, u4 = lane & 4;
            double w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const double send = u16 ? v[i] : v[i + 4];
                const double keep = u16 ? v[i + 4] : v[i];
                w[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
            }
            double x[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const double send = u8 ? w[i] : w[i + 2];
                const double keep = u8 ? w[i + 2] : w[i];
                x[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
            }
            double y = (u4 ? x[1] : x[0]) + __shfl_xor_sync(0xffffffffu, u4 ? x[0] : x[1], 4);
            y += __shfl_xor_sync(0xffffffffu, y, 2);
            y += __shfl_xor_sync(0xffffffffu, y, 1);
            const int g = lane & 3;
            const double t1 = __shfl_sync(0xffffffffu, y, 8 * g);
            const double t2 = __shfl_sync(0xffffffffu, y, 8 * g + 4);
            if ((lane >> 2) == bb) { my1 = t1; my2 = t2; }
        }
        const int bb = lane >> 2, g = lane & 3;
        const int j = jb + bb;
        if (j < j1 && g < G) {
            const int nj = min(c.bs, L - j * c.bs);
            double sc = log((double)nj) + my1;
            if (!first_order) sc += log1p(0.5 * my2);
            bool valid = false;                 // ok[] indexed by a compile-time bb
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k == bb) valid = ok[k];
            scores[((int64_t)b * c.hq + h * G + g) * c.mbp + j] = valid ? (float)sc : -SPLA_INF;
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
                                                             int kcap) {
    extern __shared__ __align__(16) unsigned char smem_sel[];
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem_sel);        // [mbp padded]
    __shared__ int hist[kBins];
    __shared__ uint32_t cand_key[kCandCap];
    __shared__ int cand_idx[kCandCap];
    __shared__ int tmp[40];
    __shared__ unsigned long long s_lo, s_hi;
    __shared__ int s_krem, s_cnt, s_done, s_mode, s_ncand;
    __shared__ uint32_t s_min, s_max;

    const int b = blockIdx.x / c.hq, hq = blockIdx.x % c.hq;
    const int tid = threadIdx.x;
    int32_t L = c.lens[b];
    L = max(0, min(L, c.mbp * c.bs));
    const int nb = (L + c.bs - 1) / c.bs;
    const float* sc = scores + ((int64_t)b * c.hq + hq) * c.mbp;
    // each thread owns P consecutive blocks, P a multiple of 32 (whole bitset words)
    const int P = max(32, ((nb + kSelThreads * 32 - 1) / (kSelThreads * 32)) * 32);
    const int own0 = tid * P, own1 = min(nb, own0 + P);

    const int fs = min(n_sink, nb), fl0 = max(0, nb - n_local);
    auto forced = [&](int j) { return j < fs || j >= fl0; };
    int nforced = fs + (nb - fl0);
    if (fl0 < fs) nforced = nb;                     // overlapping ranges
    const int ncand = nb - nforced;
    const bool take_all = ncand <= top_k;

    if (tid == 0) { s_min = 0xffffffffu; s_max = 0u; }
    __syncthreads();
    uint32_t lmin = 0xffffffffu, lmax = 0u;
    for (int j = own0; j < own1; ++j) {
        uint32_t k = forced(j) ? 0u : ordered_key(sc[j]);
        keys[j] = k;
        if (k) { lmin = min(lmin, k); lmax = max(lmax, k); }
    }
    if (!take_all) {
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
        }
        __syncthreads();
        for (int pass = 0; pass < 8 && !s_done; ++pass) {
            const unsigned long long lo = s_lo, hi = s_hi;
            int shift = 0;
            while (((hi - lo - 1ull) >> shift) >= (unsigned long long)kBins) ++shift;
            const int nbins = (int)((hi - lo - 1ull) >> shift) + 1;
            for (int i = tid; i < nbins; i += kSelThreads) hist[i] = 0;
            __syncthreads();
            for (int j = own0; j < own1; ++j) {
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
            // every key in [lo, hi) is selected: mark them above the final threshold
            for (int j = own0; j < own1; ++j)
                if (keys[j] >= lo && keys[j] < hi) keys[j] = 0xffffffffu;
        } else if (s_mode == 2) {
            for (int j = own0; j < own1; ++j)
                if (keys[j] >= lo && keys[j] < hi) {
                    const int p = atomicAdd(&s_ncand, 1);
                    if (p < kCandCap) { cand_key[p] = keys[j]; cand_idx[p] = j; }
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
            // equal keys: the krem lowest indices among keys == lo
            int cnt = 0;
            for (int j = own0; j < own1; ++j) cnt += (keys[j] == lo);
            int r = block_excl_scan(cnt, tmp, nullptr);
            for (int j = own0; j < own1; ++j)
                if (keys[j] == lo) {
                    if (r < krem) keys[j] = 0xffffffffu;
                    ++r;
                }
        }
        __syncthreads();
    }

    // flags -> bitset words, list positions
    const unsigned long long thr = take_all ? 0ull : s_hi;
    int cnt = 0;
    uint32_t* hb = bits + ((int64_t)b * c.hq + hq) * nw;
    for (int w0 = own0; w0 < own0 + P && w0 < nb; w0 += 32) {
        uint32_t word = 0u;
        for (int u = 0; u < 32; ++u) {
            const int j = w0 + u;
            if (j < nb && (take_all || forced(j) || (unsigned long long)keys[j] >= thr))
                word |= 1u << u;
        }
        hb[w0 >> 5] = word;
        cnt += __popc(word);
    }
    int total;
    int pos = block_excl_scan(cnt, tmp, &total);
    if (sel_idx) {
        int32_t* out = sel_idx + ((int64_t)b * c.hq + hq) * kcap;
        for (int w0 = own0; w0 < own0 + P && w0 < nb; w0 += 32) {
            uint32_t word = hb[w0 >> 5];
            while (word) {
                const int u = __ffs(word) - 1;
                if (pos < kcap) out[pos] = w0 + u;
                ++pos;
                word &= word - 1u;
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
            score_kernel<128, __nv_bfloat16><<<grid, 256, 0, s>>>(c, (const __nv_bfloat16*)q, scale,
                                                                 first_order, scores, chunk, status);
        else
            score_kernel<64, __nv_bfloat16><<<grid, 256, 0, s>>>(c, (const __nv_bfloat16*)q, scale,
                                                                first_order, scores, chunk, status);
    } else {
        if (c.d == 128)
            score_kernel<128, float><<<grid, 256, 0, s>>>(c, (const float*)q, scale, first_order,
                                                         scores, chunk, status);
        else
            score_kernel<64, float><<<grid, 256, 0, s>>>(c, (const float*)q, scale, first_order,
                                                        scores, chunk, status);
    }
    return cudaGetLastError();
}

cudaError_t launch_select(const CacheView& c, int top_k, int n_sink, int n_local,
                          const float* scores, uint32_t* bits, int nw, int32_t* nsel,
                          int32_t* sel_idx, int kcap, cudaStream_t s) {
    const size_t smem = (size_t)((c.mbp + 31) / 32) * 32 * sizeof(uint32_t);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(select_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    select_kernel<<<c.batch * c.hq, kSelThreads, smem, s>>>(c, top_k, n_sink, n_local, scores,
                                                            bits, nw, nsel, sel_idx, kcap);
    return cudaGetLastError();
}

}  // namespace spla
