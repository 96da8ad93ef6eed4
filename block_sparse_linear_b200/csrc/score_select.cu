// a1 + a2 -- block scoring and top-k selection (SPLA technical summary,
// gist.science, section 2.1: the block relevance is the integrated attention
// mass of its tokens, approximated around the block mean by
// exp(q.kbar)(1 + 1/2 q^T diag(sigma^2) q); the blocks with the largest
// estimates are attended exactly).
//
// score_kernel  grid (chunks + 1, batch*Hkv), 4 compute warps + 1 producer.
//               Streams each block's statistics (1 KiB at d=128, stored in
//               logical block order, so a CTA's range is contiguous) once per
//               KV head through a 4-stage ring of 16 KiB bulk copies (TMA, no
//               multicast), and scores every block for all G query heads of
//               the group: lanes split the head dimension, form the 16 fp64
//               partial dot products (2 blocks x 4 heads x 2 orders) and reduce
//               them across lanes with a transposing butterfly that leaves
//               value l in lanes l and l+16. The extra CTA of each group
//               computes the global linear-attention readout N, D (it needs no
//               selection).
// select_kernel grid (batch*Hq), 512 threads. Exact top-k by key-space
//               bucketing: 2048 linear buckets over the live key range, the
//               bucket holding the k-th key is refined until few candidates
//               remain, which are ranked pairwise (ties -> lower block index).
//               Writes a per-head selection bitset (warp ballots over 32
//               consecutive blocks), the sorted block list and its length.
#include "common.cuh"

namespace spla {

constexpr int kScoreBatch = 2;         // blocks a warp reduces together

// 16 values per lane -> lanes l and l^16 end with the warp-wide sum of value
// (l & 15) (fp64). At each level a lane keeps the half of its values whose index
// has the lane's bit set (or clear) and adds the partner's copy of that half.
__device__ __forceinline__ double transpose_reduce16(double (&v)[16]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int m = 8; m >= 1; m >>= 1) {
        const bool up = lane & m;
#pragma unroll
        for (int i = 0; i < m; ++i) {
            const double send = up ? v[i] : v[i + m];
            const double keep = up ? v[i + m] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 16);
}

constexpr int kReadoutWarps = 4;       // warps of the score CTA that compute the readout

// Global linear-attention readout of one (sequence, KV head) for its G query
// heads (linear attention over all blocks, technical summary section 2.2):
// N[g][j] = sum_i a_g,i S[i][j], D[g] = sum_i a_g,i z_i with
// a_g,i = exp(q_g,i + m_i - c_g), c_g = max_i (q_g,i + m_i). Warps split the rows.
template <int D, typename T>
__device__ void global_readout(const CacheView& c, const T* __restrict__ q, int b, int h,
                               float* __restrict__ gread, float* sm) {
    const int G = c.group, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int nwarp = kReadoutWarps;   // the calling threads: warps 0..nwarp-1
    float* aw = sm;                 // [4][D]
    float* red = aw + 4 * D;        // [nwarp][4][D + 1]
    const float* mrow = c.m + ((int64_t)b * c.hkv + h) * D;
    for (int e = threadIdx.x; e < 4 * D; e += nwarp * 32) {
        const int g = e / D, i = e % D;
        aw[e] = (g < G) ? to_f(q[((int64_t)b * c.hq + h * G + g) * D + i]) + mrow[i] : -SPLA_INF;
    }
    asm volatile("bar.sync 1, %0;" :: "r"(nwarp * 32));
    if (warp < G) {
        float mx = -SPLA_INF;
        for (int i = lane; i < D; i += 32) mx = fmaxf(mx, aw[warp * D + i]);
        mx = warp_max(mx);
        __syncwarp();
        for (int i = lane; i < D; i += 32) aw[warp * D + i] = expf(aw[warp * D + i] - mx);
    }
    asm volatile("bar.sync 1, %0;" :: "r"(nwarp * 32));
    const float* Sg = c.S + ((int64_t)b * c.hkv + h) * D * D;
    const float* zg = c.z + ((int64_t)b * c.hkv + h) * D;
    constexpr int CPL = D / 32;     // columns per lane
    float acc[4][CPL], dacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int u = 0; u < CPL; ++u) acc[g][u] = 0.f;
    const int rows = D / nwarp;
#pragma unroll 4
    for (int r = 0; r < rows; ++r) {
        const int i = warp * rows + r;
        float sv[CPL];
#pragma unroll
        for (int u = 0; u < CPL; ++u) sv[u] = __ldg(Sg + (int64_t)i * D + lane + 32 * u);
        const float zi = __ldg(zg + i);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            if (g < G) {
                const float ag = aw[g * D + i];
#pragma unroll
                for (int u = 0; u < CPL; ++u) acc[g][u] = fmaf(ag, sv[u], acc[g][u]);
                dacc[g] = fmaf(ag, zi, dacc[g]);
            }
        }
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) {
#pragma unroll
        for (int u = 0; u < CPL; ++u) red[(warp * 4 + g) * (D + 1) + lane + 32 * u] = acc[g][u];
        if (lane == 0) red[(warp * 4 + g) * (D + 1) + D] = dacc[g];
    }
    asm volatile("bar.sync 1, %0;" :: "r"(nwarp * 32));
    float* out = gread + ((int64_t)b * c.hkv + h) * G * (D + 4);
    for (int e = threadIdx.x; e < G * (D + 1); e += nwarp * 32) {
        const int g = e / (D + 1), j = e % (D + 1);
        float t = 0.f;
        for (int w = 0; w < nwarp; ++w) t += red[(w * 4 + g) * (D + 1) + j];
        out[g * (D + 4) + j] = t;
    }
}

// Grid (chunks + 1, batch*Hkv): CTAs x < chunks score a contiguous range of
// blocks, CTA x == chunks computes the group's global readout. A group's
// statistics are contiguous (logical block order), so the producer warp moves a
// whole stage of kScoreStageBlocks blocks with one bulk copy; the four compute
// warps take kScoreStageBlocks/4 blocks each, two at a time.
constexpr int kScoreStageBlocks = 16;
constexpr int kScoreStages = 4;
constexpr int kScoreWarps = 4;

template <int D, typename T>
__global__ void __launch_bounds__((kScoreWarps + 1) * 32, 3)
score_kernel(CacheView c, const T* __restrict__ q, double scale, int first_order,
             float* __restrict__ scores, int chunk, int nchunks, float* __restrict__ gread,
             int32_t* status) {
    constexpr int DPL = D / 32;                    // dimensions per lane: 2 or 4
    constexpr int REC = 2 * D;                     // floats of one block's statistics
    constexpr int STAGE = kScoreStageBlocks * REC; // floats per ring stage
    extern __shared__ __align__(128) float smem_score[];
    __shared__ uint64_t full[kScoreStages], empty[kScoreStages];
    const int b = blockIdx.y / c.hkv, h = blockIdx.y % c.hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_trigger();
    pdl_wait();
    if ((int)blockIdx.x == nchunks) {
        static_assert(kReadoutWarps <= kScoreWarps, "readout warps");
        if (threadIdx.x < kReadoutWarps * 32) global_readout<D, T>(c, q, b, h, gread, smem_score);
        return;
    }
    int32_t L = c.lens[b];
    if (L < 0 || L > c.mbp * c.bs) {
        if (blockIdx.x == 0 && threadIdx.x == 0 && h == 0) set_status(status, SPLA_DEV_CAPACITY);
        L = max(0, min(L, c.mbp * c.bs));
    }
    const int nb = (L + c.bs - 1) / c.bs;
    const int j0 = blockIdx.x * chunk;
    if (j0 >= nb) return;
    const int j1 = min(nb, j0 + chunk);
    const int nstage = (j1 - j0 + kScoreStageBlocks - 1) / kScoreStageBlocks;
    const int G = c.group;
    const float* src = c.stats + (((int64_t)b * c.hkv + h) * c.mbp + j0) * REC;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kScoreStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kScoreWarps);
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kScoreWarps) {
        // ---------------- producer
        if (lane == 0) {
            for (int t = 0; t < nstage; ++t) {
                const int st = t % kScoreStages;
                if (t >= kScoreStages && !mbar_wait_bounded(&empty[st], ((t / kScoreStages) - 1) & 1)) {
                    set_status(status, SPLA_DEV_TIMEOUT);
                    break;
                }
                const int nblk = min(kScoreStageBlocks, j1 - j0 - t * kScoreStageBlocks);
                const uint32_t bytes = (uint32_t)nblk * REC * 4;
                mbar_arrive_expect_tx(&full[st], bytes);
                bulk_load(smem_score + st * STAGE, src + (int64_t)t * STAGE, bytes, &full[st]);
            }
        }
        return;
    }

    // ---------------- compute warps
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
    constexpr int PER_WARP = kScoreStageBlocks / kScoreWarps;   // blocks of a stage per warp
    const double log_bs = log((double)c.bs);
    for (int t = 0; t < nstage; ++t) {
        const int st = t % kScoreStages;
        if (!mbar_wait_bounded(&full[st], (t / kScoreStages) & 1)) {
            set_status(status, SPLA_DEV_TIMEOUT);
            break;
        }
        const float* sb = smem_score + st * STAGE;
#pragma unroll
        for (int bb = 0; bb < PER_WARP; bb += kScoreBatch) {
            double v[8 * kScoreBatch];
#pragma unroll
            for (int k = 0; k < kScoreBatch; ++k) {
                const float* rec = sb + (warp * PER_WARP + bb + k) * REC;
                float mu[DPL], va[DPL];
                if constexpr (DPL == 4) {
                    const float4 m4 = *reinterpret_cast<const float4*>(rec + lane * 4);
                    const float4 v4 = *reinterpret_cast<const float4*>(rec + D + lane * 4);
                    mu[0] = m4.x; mu[1] = m4.y; mu[2] = m4.z; mu[3] = m4.w;
                    va[0] = v4.x; va[1] = v4.y; va[2] = v4.z; va[3] = v4.w;
                } else {
                    const float2 m2 = *reinterpret_cast<const float2*>(rec + lane * 2);
                    const float2 v2 = *reinterpret_cast<const float2*>(rec + D + lane * 2);
                    mu[0] = m2.x; mu[1] = m2.y;
                    va[0] = v2.x; va[1] = v2.y;
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    double s1 = 0.0, s2 = 0.0;
#pragma unroll
                    for (int u = 0; u < DPL; ++u) {
                        s1 = fma(qd[g][u], (double)mu[u], s1);
                        s2 = fma(q2[g][u], (double)va[u], s2);
                    }
                    v[8 * k + 2 * g] = s1;
                    v[8 * k + 2 * g + 1] = s2;
                }
            }
            const double tot = transpose_reduce16(v);
            const double t2 = __shfl_down_sync(0xffffffffu, tot, 1);
            const int k = (lane >> 3) & 1, g = (lane >> 1) & 3;
            const int j = j0 + t * kScoreStageBlocks + warp * PER_WARP + bb + k;
            if (lane < 16 && !(lane & 1) && g < G && j < j1) {
                const int nj = min(c.bs, L - j * c.bs);
                // log n_j: a constant except for a sequence's last block
                double sc = ((nj == c.bs) ? log_bs : log((double)nj)) + tot;
                if (!first_order) {
                    // log1p in fp32 where it is accurate to ~6e-8 absolute (argument <= 1)
                    const double x = 0.5 * t2;
                    sc += (x <= 1.0) ? (double)log1pf((float)x) : log1p(x);
                }
                scores[((int64_t)b * c.hq + h * G + g) * c.mbp + j] = (float)sc;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
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
    __shared__ int wpre[SPLA_MAX_BLOCKS_PER_SEQ / 32];             // per-word counts, then prefixes
    __shared__ uint32_t cand_key[kCandCap];
    __shared__ int cand_idx[kCandCap];
    __shared__ int tmp[40];
    __shared__ unsigned long long s_lo, s_hi;
    __shared__ int s_krem, s_cnt, s_done, s_mode, s_ncand, s_total;
    __shared__ uint32_t s_min, s_max;

    const int b = blockIdx.x / c.hq, hq = blockIdx.x % c.hq;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_trigger();
    pdl_wait();
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

template <int D, typename T>
static cudaError_t launch_score_t(const CacheView& c, const void* q, double scale, int first_order,
                                  float* scores, int chunk, float* gread, int32_t* status,
                                  cudaStream_t s) {
    const int nchunks = (c.mbp + chunk - 1) / chunk;
    const size_t ring = (size_t)kScoreStages * kScoreStageBlocks * 2 * D * sizeof(float);
    const size_t rd = (size_t)(4 * D + kScoreWarps * 4 * (D + 1)) * sizeof(float);
    const size_t smem = ring > rd ? ring : rd;
    cudaError_t e = cudaFuncSetAttribute(score_kernel<D, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(score_kernel<D, T>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    dim3 grid(nchunks + 1, c.batch * c.hkv);
    return launch_pdl(score_kernel<D, T>, grid, dim3((kScoreWarps + 1) * 32), smem, s, c,
                      (const T*)q, scale, first_order, scores, chunk, nchunks, gread, status);
}

cudaError_t launch_score(const CacheView& c, int dtype, const void* q, double scale,
                         int first_order, float* scores, int chunk, float* gread,
                         int32_t* status, cudaStream_t s) {
    if (dtype == SPLA_BF16)
        return c.d == 128 ? launch_score_t<128, __nv_bfloat16>(c, q, scale, first_order, scores, chunk, gread, status, s)
                          : launch_score_t<64, __nv_bfloat16>(c, q, scale, first_order, scores, chunk, gread, status, s);
    return c.d == 128 ? launch_score_t<128, float>(c, q, scale, first_order, scores, chunk, gread, status, s)
                      : launch_score_t<64, float>(c, q, scale, first_order, scores, chunk, gread, status, s);
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
    return launch_pdl(select_kernel, dim3(c.batch * c.hq), dim3(kSelThreads), smem, s, c, top_k,
                      n_sink, n_local, scores, bits, nw, nsel, sel_idx, kcap);
}

}  // namespace spla
