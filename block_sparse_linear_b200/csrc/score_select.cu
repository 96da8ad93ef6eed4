// a1 + a2 -- block scoring and top-k selection (SPLA technical summary,
// gist.science, section 2.1: the block relevance is the integrated attention
// mass of its tokens, approximated around the block mean by
// exp(q.kbar)(1 + 1/2 q^T diag(sigma^2) q); the blocks with the largest
// estimates are attended exactly).
//
// score_kernel  persistent grid (2 CTAs of 4 warp pairs per SM); every pair is
//               its own TMA pipeline over equal 32 KiB items: 32-block tiles of
//               the statistics (fp64 tensor-core dot products with the means and
//               the variances) and row ranges of the global state S for the
//               linear-attention readout N, D that the combine step subtracts
//               from.
// select_kernel grid (batch*Hq), 512 threads (1024 past 4096 blocks per
//               sequence). Exact top-k: 2048 buckets linear in the score value,
//               everything above the bucket holding the k-th key kept, that
//               bucket's keys ranked pairwise (ties -> lower block index); a
//               non-finite range or a crowded bucket falls back to key-space
//               buckets refined pass by pass. Writes a per-head selection bitset
//               (warp ballots over 32 consecutive blocks), the sorted block list
//               and its length.
#include "common.cuh"

namespace spla {

// ------------------------------------------------------------------ scoring
// One launch works through a list of equal-sized items, taken by the warp pairs
// of a persistent grid (pair p of NP takes items p, p + NP, ...):
//   items [0, groups*RP)       global readout of one (sequence, KV head) group,
//                              part p of RP row ranges of S (RP = 2 at d = 128);
//   items groups*RP + gi*ntile + t
//                              scores of blocks 32t .. 32t+31 of group gi.
// Each pair is its own pipeline: lane 0 of its first warp keeps kScoreRing
// stages of 8 KiB in flight on the pair's mbarriers; both warps consume every
// stage (each its half of the blocks, or of the readout columns) and meet on
// the pair's named barrier before the stage is refilled. Two warps per stage
// keep the dependent fp64 chains of a stage short.
//
// Score tile: the statistics are a 2-D fp32 tensor [groups*mbp rows][2d] (mean,
// then variance, logical block order); one stage is two 32 x 32 boxes (mean and
// variance of 32 dimensions of 32 blocks) with 128-byte swizzle. The dot
// products run on the fp64 tensor cores (mma m8n8k4 f64): A = 8 blocks x 4
// dimensions of statistics, B = 4 dimensions x 8 columns, the columns being
// q'_g (g < 4) and q'_g^2 (g >= 4), q' = q * softmax_scale (columns past G
// are 0). Mean tiles accumulate into one C, variance tiles into another, and
// the useful halves (mean x q', variance x q'^2) are paired across lanes at
// the end. Rows of an A fragment are blocks r/2 + 4(r%2) of an 8-block group,
// which keeps every quarter warp's 16-byte reads on distinct bank groups under
// the swizzle; warp h of a pair takes the 8-block groups 2h and 2h + 1.
//
// Readout part: N[g][j] += sum_i a_g,i S[i][j], D[g] += sum_i a_g,i z_i over
// its rows i, with a_g,i = exp(q_g,i + m_i - c_g), c_g = max over all i of
// q_g,i + m_i (the same in every part, so the parts add). S rows arrive by 1-D
// bulk copies; warp h of the pair owns columns [h d/2, (h+1) d/2).
//
// Nothing on the streaming path is read with ordinary loads: while the memory
// system is saturated with bulk traffic those take microseconds to return. An
// item's query rows (and m, z for a readout) arrive by bulk copy on a second
// per-pair barrier, issued with the item's first stage; sequence lengths are
// read into shared memory once at the start.
constexpr int kScorePairs = 4;          // warp pairs per CTA
constexpr int kScoreWarps = 2 * kScorePairs;
constexpr int kScoreRing = 2;           // stages in flight per pair
constexpr int kScoreStage = 8192;       // bytes per stage
constexpr int kScoreCtasPerSm = 2;
constexpr int kTile = 32;               // blocks per score item
constexpr int kScoreNbSmem = 512;       // sequences whose block counts are cached in smem

template <int D>
struct ScoreShape {
    static constexpr int kTileStages = D / 32;                              // 32 dims per stage
    static constexpr int kReadoutParts = (D * D * 4) / (kTileStages * kScoreStage);
    static constexpr int kRowsPerStage = kScoreStage / (D * 4);
    static constexpr int kATab = D * 4 * 4;                                 // readout weights [D][4]
    // per-item inputs by bulk copy: the group's G query rows (up to 2 KiB), then m and z (D floats each)
    static constexpr int kQBytes = 2048;
    static constexpr int kAux = kQBytes + 2 * D * 4;
    static constexpr int kAuxPad = 1024 * ((kAux + 1023) / 1024);
    // two input buffers: item k uses buffer k % 2, so the next item's copy never
    // lands in rows the current item still reads
    static constexpr int kPairBytes = kScoreRing * kScoreStage + kATab + 2 * kAuxPad;
    static constexpr int kSmem = kScorePairs * kPairBytes + 1024;           // + alignment
    static_assert(kReadoutParts >= 1 && kReadoutParts * kTileStages * kRowsPerStage == D, "parts");
    static_assert(kPairBytes % 1024 == 0, "ring alignment for the 128B swizzle");
};

// D(8x8, f64) += A(8x4, row) * B(4x8, col); per lane a = A[lane/4][lane%4],
// b = B[lane%4][lane/4], c = D[lane/4][2(lane%4) .. +1].
__device__ __forceinline__ void dmma_884(double (&c)[2], double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                 : "+d"(c[0]), "+d"(c[1]) : "d"(a), "d"(b));
}

// log n for n = 0 .. 128 (entry 0 unused): the log n_j term of a partial block.
__constant__ double c_log_n[129] = {0.0, 0.0, 0.6931471805599453, 1.0986122886681098, 1.3862943611198906, 1.6094379124341003, 1.791759469228055, 1.9459101490553132, 2.0794415416798357, 2.1972245773362196, 2.302585092994046, 2.3978952727983707, 2.4849066497880004, 2.5649493574615367, 2.6390573296152584, 2.70805020110221, 2.772588722239781, 2.833213344056216, 2.8903717578961645, 2.9444389791664403, 2.995732273553991, 3.044522437723423, 3.091042453358316, 3.1354942159291497, 3.1780538303479458, 3.2188758248682006, 3.258096538021482, 3.295836866004329, 3.332204510175204, 3.367295829986474, 3.4011973816621555, 3.4339872044851463, 3.4657359027997265, 3.4965075614664802, 3.5263605246161616, 3.5553480614894135, 3.58351893845611, 3.6109179126442243, 3.6375861597263857, 3.6635616461296463, 3.6888794541139363, 3.713572066704308, 3.7376696182833684, 3.7612001156935624, 3.784189633918261, 3.8066624897703196, 3.828641396489095, 3.8501476017100584, 3.871201010907891, 3.8918202981106265, 3.912023005428146, 3.9318256327243257, 3.9512437185814275, 3.970291913552122, 3.9889840465642745, 4.007333185232471, 4.02535169073515, 4.04305126783455, 4.060443010546419, 4.07753744390572, 4.0943445622221, 4.110873864173311, 4.127134385045092, 4.143134726391533, 4.1588830833596715, 4.174387269895637, 4.189654742026425, 4.204692619390966, 4.219507705176107, 4.23410650459726, 4.248495242049359, 4.2626798770413155, 4.276666119016055, 4.290459441148391, 4.30406509320417, 4.31748811353631, 4.330733340286331, 4.343805421853684, 4.356708826689592, 4.3694478524670215, 4.382026634673881, 4.394449154672439, 4.406719247264253, 4.418840607796598, 4.430816798843313, 4.442651256490317, 4.454347296253507, 4.465908118654584, 4.477336814478207, 4.48863636973214, 4.499809670330265, 4.51085950651685, 4.5217885770490405, 4.532599493153256, 4.543294782270004, 4.553876891600541, 4.564348191467836, 4.574710978503383, 4.584967478670572, 4.59511985013459, 4.605170185988092, 4.61512051684126, 4.624972813284271, 4.634728988229636, 4.6443908991413725, 4.653960350157523, 4.663439094112067, 4.672828834461906, 4.68213122712422, 4.6913478822291435, 4.700480365792417, 4.709530201312334, 4.718498871295094, 4.727387818712341, 4.736198448394496, 4.74493212836325, 4.7535901911063645, 4.762173934797756, 4.770684624465665, 4.77912349311153, 4.787491742782046, 4.795790545596741, 4.804021044733257, 4.812184355372417, 4.820281565605037, 4.8283137373023015, 4.836281906951478, 4.844187086458591, 4.852030263919617};

template <typename T> struct QVec;
template <> struct QVec<__nv_bfloat16> {
    // 4 consecutive bf16 values (8 bytes) as floats
    static __device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&v)[4]) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    }
};
template <> struct QVec<float> {
    static __device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
        const float4 u = *reinterpret_cast<const float4*>(p);
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    }
};

template <int D, typename T>
__global__ void __launch_bounds__(kScoreWarps * 32, kScoreCtasPerSm)
score_kernel(const __grid_constant__ CUtensorMap tstats, CacheView c, const T* __restrict__ q,
             double scale, double log_bs, int first_order, float* __restrict__ scores, int ld,
             float* __restrict__ gread, float* __restrict__ aw_out, int ntile, KernelStamps* stamps,
             int32_t* status) {
    using S = ScoreShape<D>;
    constexpr int RP = S::kReadoutParts, TS = S::kTileStages, RPS = S::kRowsPerStage;
    constexpr int CPL = D / 32;                    // rows per lane in the readout weights
    constexpr int HC = D / 2;                      // readout columns per warp
    constexpr int CPH = HC / 32;                   // readout columns per lane
    extern __shared__ unsigned char smem_raw[];
    __shared__ uint64_t full[kScorePairs][kScoreRing];
    __shared__ uint64_t qfull[kScorePairs][2];
    __shared__ int s_nb[kScoreNbSmem], s_len[kScoreNbSmem];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int pair = warp >> 1, half = warp & 1;
    // 1024-byte alignment by shared-pointer arithmetic (keeps the accesses ld.shared)
    unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    unsigned char* ring = base + pair * S::kPairBytes;
    float* at = reinterpret_cast<float*>(ring + kScoreRing * kScoreStage);    // readout [D][4]
    unsigned char* aux0 = ring + kScoreRing * kScoreStage + S::kATab;          // q rows, m, z (x2)
    uint64_t* bar = full[pair];
    uint64_t* qbar = qfull[pair];
    const int G = c.group, hkv = c.hkv, mbp = c.mbp, bs = c.bs;
    const int groups = c.batch * hkv;
    const int nread = groups * RP;
    const int nitems = nread + groups * ntile;
    const int NP = gridDim.x * kScorePairs;
    const int wp = blockIdx.x * kScorePairs + pair;
    const bool leader = half == 0 && lane == 0;     // the pair's producer thread
    const uint32_t pair_bar = 1u + (uint32_t)pair;  // named barrier of the pair (0 is __syncthreads)
    auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;" :: "r"(pair_bar) : "memory"); };

    pdl_trigger();
    if (threadIdx.x == 0) prefetch_tmap(&tstats);
    // Before the dependency wait, warm L2 with the first stage of this pair's first
    // score item (its two boxes). A prefetch only: the copies that use the data go out
    // after the wait and read L2, which holds whatever the append kernels wrote. Those
    // first copies then hit L2 instead of queueing behind every pair's first request.
    if (leader) {
        for (int i = wp; i < nitems; i += NP) {
            if (i < nread) continue;
            const int r = i - nread, gi = r / ntile, t = r % ntile;
            const int y = gi * mbp + t * kTile;
            tma_prefetch_2d(&tstats, 0, y);
            tma_prefetch_2d(&tstats, D, y);
            break;
        }
    }
    if (leader) {
        for (int s = 0; s < kScoreRing; ++s) mbar_init(&bar[s], 1);
        mbar_init(&qbar[0], 1);
        mbar_init(&qbar[1], 1);
        fence_barrier_init();
    }
    pdl_wait();          // statistics, state and lengths come from the append kernels
    if (threadIdx.x == 0) stamp_first(stamps, kStampScore);
    for (int b = threadIdx.x; b < min(c.batch, kScoreNbSmem); b += blockDim.x) {
        const int32_t L = c.lens[b];
        if (blockIdx.x == 0 && (L < 0 || L > mbp * bs)) set_status(status, SPLA_DEV_CAPACITY);
        s_len[b] = max(0, min(L, mbp * bs));
        s_nb[b] = (s_len[b] + bs - 1) / bs;
    }
    __syncthreads();
    auto len_of = [&](int b) {
        return b < kScoreNbSmem ? s_len[b] : max(0, min(c.lens[b], mbp * bs));
    };
    auto nb_of = [&](int b) {
        if (b < kScoreNbSmem) return s_nb[b];
        return (len_of(b) + bs - 1) / bs;
    };
    // next non-empty item at or after i in this pair's sequence
    auto next_item = [&](int i) {
        for (; i < nitems; i += NP) {
            if (i < nread) return i;
            const int r = i - nread, gi = r / ntile, t = r % ntile;
            if (t * kTile < nb_of(gi / hkv)) return i;
        }
        return nitems;
    };

    // ---- producer state (the leader): item, stage within it, stages issued
    int pi = next_item(wp), ps = 0, fi = 0, pk = 0;     // pk: items issued
    // the current item's source, worked out at its first stage: the statistics row of
    // its tile, or its part of S
    int py = 0;
    const float* psrc = nullptr;
    auto issue = [&]() {
        if (pi >= nitems) return;
        const int slot = fi % kScoreRing;
        unsigned char* dst = ring + slot * kScoreStage;
        if (ps == 0) {
            // the item's query rows (and m, z for a readout) on the item barrier
            int gi;
            if (pi < nread) {
                gi = pi / RP;
                psrc = c.S + (int64_t)gi * D * D + (int64_t)(pi % RP) * TS * RPS * D;
            } else {
                const int r = pi - nread;
                gi = r / ntile;
                py = gi * mbp + (r - gi * ntile) * kTile;
            }
            const int b = gi / hkv, h = gi - (gi / hkv) * hkv;
            const uint32_t qb = (uint32_t)(G * D * sizeof(T));
            unsigned char* ax = aux0 + (pk & 1) * S::kAuxPad;
            uint64_t* qb_bar = &qbar[pk & 1];
            ++pk;
            mbar_arrive_expect_tx(qb_bar, qb + (pi < nread ? 2u * D * 4u : 0u));
            bulk_load(ax, q + ((int64_t)b * c.hq + h * G) * D, qb, qb_bar);
            if (pi < nread) {
                bulk_load(ax + S::kQBytes, c.m + (int64_t)gi * D, D * 4, qb_bar);
                bulk_load(ax + S::kQBytes + D * 4, c.z + (int64_t)gi * D, D * 4, qb_bar);
            }
        }
        mbar_arrive_expect_tx(&bar[slot], kScoreStage);
        if (pi < nread) {
            bulk_load(dst, psrc + (int64_t)ps * RPS * D, kScoreStage, &bar[slot]);
        } else {
            tma_load_2d(dst, &tstats, &bar[slot], ps * 32, py);
            tma_load_2d(dst + kScoreStage / 2, &tstats, &bar[slot], D + ps * 32, py);
        }
        ++fi;
        if (++ps == TS) {
            ps = 0;
            pi = next_item(pi + NP);
        }
    };
    if (leader)
        for (int s = 0; s < kScoreRing; ++s) issue();

    int f = 0;                 // stages consumed
    int nq = 0;                // items started: buffer nq % 2, its phase (nq / 2) % 2
    // after a failed wait the leader waits (bounded) for every copy it has in flight
    auto drain = [&](int q_from) {
        set_status(status, SPLA_DEV_TIMEOUT);
        for (int k = f; k < fi; ++k) mbar_wait_bounded(&bar[k % kScoreRing], (k / kScoreRing) & 1);
        for (int k = q_from; k < pk; ++k) mbar_wait_bounded(&qbar[k & 1], (k >> 1) & 1);
    };
    // every lane of the warp agrees on the outcome of a wait; a warp that gives up
    // returns, and its partner's next wait on a copy that never comes gives up too
    auto wait_stage = [&](int slot) -> bool {
        return __all_sync(0xffffffffu, mbar_wait_bounded(&bar[slot], (f / kScoreRing) & 1));
    };
    const T* qs = nullptr;
    const float* ms = nullptr;
    const float* zs_ = nullptr;
    auto wait_item = [&]() -> bool {
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&qbar[nq & 1], (nq >> 1) & 1));
        const unsigned char* ax = aux0 + (nq & 1) * S::kAuxPad;
        qs = reinterpret_cast<const T*>(ax);
        ms = reinterpret_cast<const float*>(ax + S::kQBytes);
        zs_ = ms + D;
        ++nq;
        return ok;
    };
    const int kq = lane & 3, rq = lane >> 2;
    const int prow = (rq >> 1) + 4 * (rq & 1);          // block row of A row rq in a group of 8
    // swizzled offsets of this lane's A fragments: [8-block group of this warp][k half]
    uint32_t aoff[2][2];
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) aoff[mi][hf] = swz128(8 * (2 * half + mi) + prow, 4 * hf + kq);
    // both warps of a pair take every wait's outcome together: a failed wait sets
    // the pair's flag, and after the next pair barrier both leave
    __shared__ int s_fail[kScorePairs];
    if (leader) s_fail[pair] = 0;
    pair_sync();
    // q_from: the first item copy that may still be in flight
    auto agree = [&](bool ok, int q_from) -> bool {
        if (!ok && lane == 0) s_fail[pair] = 1;
        pair_sync();
        if (s_fail[pair]) {
            if (leader) drain(q_from);
            return false;
        }
        return true;
    };

    for (int i = next_item(wp); i < nitems; i = next_item(i + NP)) {
        if (i < nread) {
            // ---------------- global readout, rows of part `part`, columns of this warp
            const int gi = i / RP, part = i % RP;
            float dsum[4];
            {
                const bool okq = wait_item();     // advances nq
                if (!agree(okq, nq - 1)) return;
            }
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                dsum[g] = 0.f;
                if (g < G) {
                    float v[CPL], mx = -SPLA_INF;
#pragma unroll
                    for (int u = 0; u < CPL; ++u) {
                        const int r = lane + 32 * u;
                        v[u] = to_f(qs[g * D + r]) + ms[r];
                        mx = fmaxf(mx, v[u]);
                    }
                    mx = warp_max(mx);
                    float zs = 0.f;
#pragma unroll
                    for (int u = 0; u < CPL; ++u) {
                        const int r = lane + 32 * u;
                        const float a = (mx == -SPLA_INF) ? 0.f : expf(v[u] - mx);
                        // each warp writes its half of the rows; both read all of them
                        if ((r >= HC) == (half == 1)) at[r * 4 + g] = a;
                        if (r / (D / RP) == part) zs = fmaf(a, zs_[r], zs);
                    }
                    dsum[g] = warp_sum(zs);
                } else {
#pragma unroll
                    for (int u = 0; u < CPL; ++u) {
                        const int r = lane + 32 * u;
                        if ((r >= HC) == (half == 1)) at[r * 4 + g] = 0.f;
                    }
                }
            }
            pair_sync();                   // the whole weight table is written
            if (part == 0) {
                // the decode kernels weight phi(k) with the same a_g,i
                float4* awg = reinterpret_cast<float4*>(aw_out + (int64_t)gi * D * 4);
                for (int r = half * HC + lane; r < (half + 1) * HC; r += 32)
                    awg[r] = *reinterpret_cast<const float4*>(at + r * 4);
            }
            float acc[4][CPH];
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
                for (int u = 0; u < CPH; ++u) acc[g][u] = 0.f;
#pragma unroll 1
            for (int s = 0; s < TS; ++s, ++f) {
                const int slot = f % kScoreRing;
                const bool ok = wait_stage(slot);
                if (ok) {
                    const float* sm = reinterpret_cast<const float*>(ring + slot * kScoreStage);
                    const int row0 = (part * TS + s) * RPS;
#pragma unroll 4
                    for (int r = 0; r < RPS; ++r) {
                        const float4 a4 = *reinterpret_cast<const float4*>(at + (row0 + r) * 4);
                        float sv[CPH];
                        if constexpr (CPH == 2) {
                            const float2 t2 = *reinterpret_cast<const float2*>(sm + r * D + half * HC + lane * 2);
                            sv[0] = t2.x; sv[1] = t2.y;
                        } else {
                            sv[0] = sm[r * D + half * HC + lane];
                        }
                        const float ag[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                        for (int g = 0; g < 4; ++g)
#pragma unroll
                            for (int u = 0; u < CPH; ++u) acc[g][u] = fmaf(ag[g], sv[u], acc[g][u]);
                    }
                }
                if (!agree(ok, nq)) return;
                if (leader) issue();
            }
            float* out = gread + ((int64_t)gi * RP + part) * G * (D + 4);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                if (g < G) {
#pragma unroll
                    for (int u = 0; u < CPH; ++u) out[g * (D + 4) + half * HC + lane * CPH + u] = acc[g][u];
                    if (half == 0 && lane == 0) out[g * (D + 4) + D] = dsum[g];
                }
            }
            continue;
        }
        // ---------------- score tile: this warp's 16 of the 32 blocks
        const int r = i - nread, gi = r / ntile, t = r % ntile;
        const int b = gi / hkv, h = gi % hkv;
        {
            const bool okq = wait_item();         // advances nq
            if (!agree(okq, nq - 1)) return;
        }
        double cm[2][2], cs[2][2];
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) cm[mi][0] = cm[mi][1] = cs[mi][0] = cs[mi][1] = 0.0;
        const int head = rq & 3;
        const bool sq = rq >= 4;
        const T* qh = qs + head * D;
        // one copy of the stage code (kept small: it runs cold at first, while the
        // memory system is saturated)
#pragma unroll 1
        for (int s = 0; s < TS; ++s, ++f) {
            // B[k][n] of k-slice (hf, u) is column n's query value at dimension
            // 32s + 16hf + 4k + u: q'_n for n < 4, q'_{n-4}^2 for n >= 4, 0 past G.
            double bq[8];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float v[4] = {0.f, 0.f, 0.f, 0.f};
                if (head < G) QVec<T>::load4(qh + 32 * s + 16 * hf + 4 * kq, v);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const double x = (double)v[u] * scale;
                    bq[hf * 4 + u] = sq ? x * x : x;
                }
            }
            const int slot = f % kScoreRing;
            const bool ok = wait_stage(slot);
            if (ok) {
                const unsigned char* st = ring + slot * kScoreStage;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float mu[2][4], va[2][4];
#pragma unroll
                    for (int mi = 0; mi < 2; ++mi) {
                        const float4 m4 = *reinterpret_cast<const float4*>(st + aoff[mi][hf]);
                        const float4 v4 = *reinterpret_cast<const float4*>(st + kScoreStage / 2 + aoff[mi][hf]);
                        mu[mi][0] = m4.x; mu[mi][1] = m4.y; mu[mi][2] = m4.z; mu[mi][3] = m4.w;
                        va[mi][0] = v4.x; va[mi][1] = v4.y; va[mi][2] = v4.z; va[mi][3] = v4.w;
                    }
                    // four independent accumulators per k-slice
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
#pragma unroll
                        for (int mi = 0; mi < 2; ++mi) {
                            dmma_884(cm[mi], (double)mu[mi][u], bq[hf * 4 + u]);
                            dmma_884(cs[mi], (double)va[mi][u], bq[hf * 4 + u]);
                        }
                    }
                }
            }
            if (!agree(ok, nq)) return;
            if (leader) issue();
        }
        // lanes kq < 2 hold mean x q' (columns 2kq, 2kq+1 = heads); their partners
        // kq + 2 hold variance x q'^2 for the same heads
        const int nbs = nb_of(b);
        const int32_t L = len_of(b);
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
            const double mine0 = (kq < 2) ? cm[mi][0] : cs[mi][0];
            const double mine1 = (kq < 2) ? cm[mi][1] : cs[mi][1];
            const double oth0 = __shfl_xor_sync(0xffffffffu, mine0, 2);
            const double oth1 = __shfl_xor_sync(0xffffffffu, mine1, 2);
            const int j = t * kTile + 8 * (2 * half + mi) + prow;
            if (kq < 2 && j < nbs) {
                const int nj = min(bs, L - j * bs);
                // log n_j: a constant except for a sequence's last block
                const double lg = (nj == bs) ? log_bs : c_log_n[nj];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int g = 2 * kq + e;
                    if (g < G) {
                        double sc = lg + (e ? mine1 : mine0);
                        if (!first_order) {
                            // fp32 log1p: within one fp32 ulp of the result, under 2.5e-7
                            // while the argument stays below e^4 - 1
                            sc += (double)log1pf((float)(0.5 * (e ? oth1 : oth0)));
                        }
                        scores[((int64_t)b * c.hq + h * G + g) * ld + j] = (float)sc;
                    }
                }
            }
        }
    }
    // (a warp that left early on a failed wait stamps nothing: the status says it failed)
    if (threadIdx.x == 0) stamp_last(stamps, kStampScore);
}

// ------------------------------------------------------------------ selection
constexpr int kBins = 2048;
constexpr int kCandCap = 256;
constexpr uint32_t kMark = 0xffffffffu;     // a selected key (only a NaN score maps here)
// threads per head: 512, or 1024 once a sequence can hold more than 4096 blocks
constexpr int kSelThreadsLong = 1024;
constexpr int kSelLongBlocks = 4096;

// The float a key was made from (the inverse of ordered_key).
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

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

// Marks (kMark) the krem largest of the nc gathered candidates: one composite per
// candidate, a larger key or an equal key at a lower block index comparing
// greater. Starts and ends on a barrier-separated state.
__device__ __forceinline__ void rank_candidates(uint32_t* keys, const uint32_t* cand_key,
                                                const int* cand_idx, unsigned long long* cand_c,
                                                int nc, int krem) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int ncp = (nc + 7) & ~7;
    for (int i = tid; i < ncp; i += nt)
        cand_c[i] = (i < nc) ? (((unsigned long long)cand_key[i] << 32) |
                                (uint32_t)~(uint32_t)cand_idx[i])
                             : 0ull;
    __syncthreads();
    for (int i = tid; i < nc; i += nt) {
        const unsigned long long mine = cand_c[i];
        int rank = 0;
        // eight candidates per step, their loads in flight together
        for (int o = 0; o < ncp; o += 8) {
            const ulonglong2 x0 = *reinterpret_cast<const ulonglong2*>(cand_c + o);
            const ulonglong2 x1 = *reinterpret_cast<const ulonglong2*>(cand_c + o + 2);
            const ulonglong2 x2 = *reinterpret_cast<const ulonglong2*>(cand_c + o + 4);
            const ulonglong2 x3 = *reinterpret_cast<const ulonglong2*>(cand_c + o + 6);
            rank += (x0.x > mine) + (x0.y > mine) + (x1.x > mine) + (x1.y > mine) +
                    (x2.x > mine) + (x2.y > mine) + (x3.x > mine) + (x3.y > mine);
        }
        if (rank < krem) keys[cand_idx[i]] = kMark;
    }
    __syncthreads();
}

// Selection of one head. Keys are the scores in a monotone uint32 order (forced
// sink and local blocks get key 0 and are always kept).
//   fast pass  2048 buckets linear in the score value over [min, max]: scores
//              spread over many buckets, so the shared-memory counters see little
//              contention; the bucket holding the k-th largest key is found by a
//              suffix scan, every key above it is marked selected, and the bucket's
//              keys (few) are ranked pairwise (ties -> lower block index).
//   refinement (a non-finite score range, or more than kCandCap keys in that
//              bucket) buckets linear in key space, narrowed pass by pass.
// Every step that reads what another warp wrote is one barrier apart; no loop
// carries a dependency through shared memory.
template <int NT, int MAXB>
__global__ void __launch_bounds__(NT) select_kernel(CacheView c, int top_k, int n_sink,
                                                    int n_local, const float* scores, int ld,
                                                    uint32_t* bits, int nw, int32_t* nsel,
                                                    int32_t* sel_idx, int kcap,
                                                    KernelStamps* stamps) {
    constexpr int kSelThreads = NT;
    constexpr int kSelWarps = NT / 32;
    constexpr int kWordsPerThread = MAXB / 32 / NT;
    constexpr int BPT = kBins / NT;             // histogram buckets per thread in the scans
    static_assert(kWordsPerThread * 32 * NT == MAXB, "bitset words per thread");
    static_assert(MAXB / NT <= 64, "candidate rounds fit a 64-bit mask");
    static_assert(BPT * NT == kBins, "buckets per thread");
    extern __shared__ __align__(16) unsigned char smem_sel[];
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem_sel);        // [mbp padded]
    __shared__ int hist[kBins];
    __shared__ int wpre[MAXB / 32];             // per-word counts, then prefixes
    __shared__ uint32_t wword[MAXB / 32];       // the bitset words
    __shared__ uint32_t cand_key[kCandCap];
    __shared__ int cand_idx[kCandCap];
    __shared__ __align__(16) unsigned long long cand_c[kCandCap];   // key << 32 | ~index
    __shared__ int tmp[40];
    __shared__ uint32_t wmn[kSelWarps], wmx[kSelWarps];
    __shared__ unsigned long long s_lo, s_hi;
    __shared__ int s_krem, s_cnt, s_done, s_mode, s_ncand, s_bstar;

    const int b = blockIdx.x / c.hq, hq = blockIdx.x % c.hq;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    // the decode kernels launch only now: before their own wait they may read what
    // the scoring kernel wrote (it has completed)
    pdl_trigger();
    if (tid == 0) stamp_first(stamps, kStampSelect);
    const float* sc = scores + ((int64_t)b * c.hq + hq) * ld;
    // the first batch of score loads goes out with the length load, bounded by the
    // capacity (entries past the sequence's blocks are loaded and ignored)
    constexpr int kKeyBatch = 8;
    float x0[kKeyBatch];
#pragma unroll
    for (int u = 0; u < kKeyBatch; ++u) {
        const int j = tid + u * kSelThreads;
        x0[u] = (j < c.mbp) ? __ldcg(sc + j) : 0.f;
    }
    int32_t L = c.lens[b];
    L = max(0, min(L, c.mbp * c.bs));
    const int nb = (L + c.bs - 1) / c.bs;
    // block j belongs to thread j % kSelThreads; rounds of kSelThreads consecutive blocks
    const int rounds = (nb + kSelThreads - 1) / kSelThreads;

    const int fs = min(n_sink, nb), fl0 = max(0, nb - n_local);
    auto forced = [&](int j) { return j < fs || j >= fl0; };
    int nforced = fs + (nb - fl0);
    if (fl0 < fs) nforced = nb;                     // overlapping ranges
    const int ncand = nb - nforced;
    const bool take_all = ncand <= top_k;

    // ---- keys, their range, and cleared bucket counters
    uint32_t lmin = 0xffffffffu, lmax = 0u;
    // kKeyBatch score loads in flight before any key is formed
    for (int j0 = tid; j0 < nb; j0 += kKeyBatch * kSelThreads) {
        float x[kKeyBatch];
#pragma unroll
        for (int u = 0; u < kKeyBatch; ++u) {
            const int j = j0 + u * kSelThreads;
            x[u] = (j0 == tid) ? x0[u] : ((j < nb) ? __ldcg(sc + j) : 0.f);
        }
#pragma unroll
        for (int u = 0; u < kKeyBatch; ++u) {
            const int j = j0 + u * kSelThreads;
            if (j < nb) {
                const uint32_t k = forced(j) ? 0u : ordered_key(x[u]);
                keys[j] = k;
                if (k) { lmin = min(lmin, k); lmax = max(lmax, k); }
            }
        }
    }
    for (int i = tid; i < kBins; i += kSelThreads) hist[i] = 0;
    if (tid == 0) { s_ncand = 0; s_bstar = -1; s_cnt = 0; s_krem = top_k; }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        lmin = min(lmin, __shfl_xor_sync(0xffffffffu, lmin, o));
        lmax = max(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    }
    if (lane == 0) { wmn[warp] = lmin; wmx[warp] = lmax; }
    __syncthreads();

    unsigned long long thr = 0ull;                  // keys >= thr are selected
    if (!take_all) {
        uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
        for (int w = 0; w < kSelWarps; ++w) { kmin = min(kmin, wmn[w]); kmax = max(kmax, wmx[w]); }
        const float fmin = key_value(kmin), fmax = key_value(kmax);
        const float span = fmax - fmin;
        // block-uniform: every thread computed the same range
        const bool fast = isfinite(fmin) && isfinite(fmax) && span > 0.f && isfinite(span);
        bool refine = !fast;
        if (fast) {
            const float scl = (float)kBins / span;
            // monotone in the key: a larger key never lands in a lower bucket
            auto fbin = [&](uint32_t k) {
                return min(kBins - 1, max(0, (int)((key_value(k) - fmin) * scl)));
            };
            // four keys per step, their loads and bucket arithmetic independent
            for (int j0 = tid; j0 < nb; j0 += 4 * kSelThreads) {
                uint32_t kk[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = j0 + u * kSelThreads;
                    kk[u] = j < nb ? keys[j] : 0u;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (kk[u]) atomicAdd(&hist[fbin(kk[u])], 1);
            }
            __syncthreads();
            // suffix scan from the top bucket; thread t covers reversed buckets [BPT t, BPT t + BPT)
            int local[BPT], lsum = 0;
#pragma unroll
            for (int u = 0; u < BPT; ++u) {
                local[u] = hist[kBins - 1 - (BPT * tid + u)];
                lsum += local[u];
            }
            const int before = block_excl_scan(lsum, tmp, nullptr);
            if (before < top_k && before + lsum >= top_k) {
                int acc = before;
#pragma unroll
                for (int u = 0; u < BPT; ++u) {
                    if (acc < top_k && acc + local[u] >= top_k) {
                        s_bstar = kBins - 1 - (BPT * tid + u);
                        s_krem = top_k - acc;        // still to take from the bucket
                        s_cnt = local[u];
                    }
                    acc += local[u];
                }
            }
            __syncthreads();
            const int bstar = s_bstar, krem = s_krem;
            if (s_cnt <= kCandCap) {
                // everything above the bucket is selected; the bucket's keys are
                // candidates, recorded per thread (bit r: round r) and placed by a scan
                unsigned long long cmask = 0ull;
                for (int r0 = 0; r0 < rounds; r0 += 4) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int r = r0 + u, j = r * kSelThreads + tid;
                        if (r < rounds && j < nb) {
                            const uint32_t k = keys[j];
                            if (k) {
                                const int bb = fbin(k);
                                if (bb > bstar) keys[j] = kMark;
                                else if (bb == bstar) cmask |= 1ull << r;
                            }
                        }
                    }
                }
                int ncnd;
                int p = block_excl_scan(__popcll(cmask), tmp, &ncnd);
                while (cmask) {
                    const int r = __ffsll((long long)cmask) - 1;
                    cmask &= cmask - 1ull;
                    const int j = r * kSelThreads + tid;
                    if (p < kCandCap) { cand_key[p] = keys[j]; cand_idx[p] = j; }
                    ++p;
                }
                __syncthreads();
                rank_candidates(keys, cand_key, cand_idx, cand_c, min(ncnd, kCandCap), krem);
                thr = kMark;
            } else {
                // key range of the crowded bucket, then key-space refinement inside it
                uint32_t bmin = 0xffffffffu, bmax = 0u;
                for (int j = tid; j < nb; j += kSelThreads) {
                    const uint32_t k = keys[j];
                    if (k && fbin(k) == bstar) { bmin = min(bmin, k); bmax = max(bmax, k); }
                }
#pragma unroll
                for (int o = 16; o; o >>= 1) {
                    bmin = min(bmin, __shfl_xor_sync(0xffffffffu, bmin, o));
                    bmax = max(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
                }
                __syncthreads();                     // every thread has read wmn / wmx
                if (lane == 0) { wmn[warp] = bmin; wmx[warp] = bmax; }
                __syncthreads();
                kmin = 0xffffffffu; kmax = 0u;
#pragma unroll
                for (int w = 0; w < kSelWarps; ++w) { kmin = min(kmin, wmn[w]); kmax = max(kmax, wmx[w]); }
                if (tid == 0) { s_lo = kmin; s_hi = (unsigned long long)kmax + 1ull; }
                refine = true;
            }
        } else if (tid == 0) {
            s_lo = kmin;
            s_hi = (unsigned long long)kmax + 1ull;
            s_krem = top_k;
        }
        if (refine) {
            if (tid == 0) { s_done = 0; s_mode = 0; }
            __syncthreads();
            for (int pass = 0; pass < 8 && !s_done; ++pass) {
                const unsigned long long lo = s_lo, hi = s_hi;
                // the smallest shift that maps [lo, hi) onto at most kBins buckets
                const unsigned long long range = hi - lo - 1ull;
                const int shift = max(0, 64 - __clzll((long long)range) - 11);
                const int nbins = (int)(range >> shift) + 1;
                for (int i = tid; i < nbins; i += kSelThreads) hist[i] = 0;
                __syncthreads();
                for (int j = tid; j < nb; j += kSelThreads) {
                    const unsigned long long k = keys[j];
                    if (k >= lo && k < hi) atomicAdd(&hist[(int)((k - lo) >> shift)], 1);
                }
                __syncthreads();
                int local[BPT], lsum = 0;
#pragma unroll
                for (int u = 0; u < BPT; ++u) {
                    const int r = BPT * tid + u;
                    local[u] = (r < nbins) ? hist[nbins - 1 - r] : 0;
                    lsum += local[u];
                }
                const int before = block_excl_scan(lsum, tmp, nullptr);
                const int krem = s_krem;
                if (before < krem && before + lsum >= krem) {
                    int acc = before;
#pragma unroll
                    for (int u = 0; u < BPT; ++u) {
                        if (acc < krem && acc + local[u] >= krem) {
                            const int bst = nbins - 1 - (BPT * tid + u);
                            const unsigned long long nlo = lo + ((unsigned long long)bst << shift);
                            unsigned long long nhi = lo + ((unsigned long long)(bst + 1) << shift);
                            if (nhi > hi) nhi = hi;
                            s_lo = nlo;
                            s_hi = nhi;
                            s_krem = krem - acc;     // still to take from [nlo, nhi)
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
                // every key in [lo, hi) is selected
                for (int j = tid; j < nb; j += kSelThreads)
                    if (keys[j] >= lo && keys[j] < hi) keys[j] = kMark;
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
                rank_candidates(keys, cand_key, cand_idx, cand_c, min(s_ncand, kCandCap), krem);
            } else {
                // equal keys: the krem lowest indices among keys == lo, in index order
                int taken = 0;
                for (int r = 0; r < rounds; ++r) {
                    const int j = r * kSelThreads + tid;
                    const bool eq = j < nb && keys[j] == lo;
                    int tot;
                    const int rank = taken + block_excl_scan(eq ? 1 : 0, tmp, &tot);
                    if (eq && rank < krem) keys[j] = kMark;
                    taken += tot;
                }
            }
            thr = hi;
        }
        __syncthreads();
    }

    // ---- flags -> bitset words (one ballot per 32 consecutive blocks), then list positions
    uint32_t* hb = bits + ((int64_t)b * c.hq + hq) * nw;
    const int nwu = (nb + 31) >> 5;
    for (int r0 = 0; r0 < rounds; r0 += 4) {
        bool sel[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = r0 + u, j = r * kSelThreads + tid;
            sel[u] = r < rounds && j < nb &&
                     (take_all || forced(j) || (unsigned long long)keys[j] >= thr);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = r0 + u;
            const uint32_t word = __ballot_sync(0xffffffffu, sel[u]);
            const int wi = r * kSelWarps + warp;
            if (lane == 0 && r < rounds && wi < nwu) {
                hb[wi] = word;
                wword[wi] = word;
                wpre[wi] = __popc(word);
            }
        }
    }
    __syncthreads();
    // exclusive scan of the word counts: thread t owns words [t * W, t * W + W)
    int total;
    {
        int cw[kWordsPerThread], v = 0;
#pragma unroll
        for (int u = 0; u < kWordsPerThread; ++u) {
            const int w = tid * kWordsPerThread + u;
            cw[u] = w < nwu ? wpre[w] : 0;
            v += cw[u];
        }
        int run = block_excl_scan(v, tmp, &total);
#pragma unroll
        for (int u = 0; u < kWordsPerThread; ++u) {
            const int w = tid * kWordsPerThread + u;
            if (w < nwu) wpre[w] = run;
            run += cw[u];
        }
    }
    __syncthreads();
    if (sel_idx) {
        int32_t* out = sel_idx + ((int64_t)b * c.hq + hq) * kcap;
        for (int r = 0; r < rounds; ++r) {
            const int j = r * kSelThreads + tid;
            const int wi = r * kSelWarps + warp;
            if (wi < nwu) {
                const uint32_t word = wword[wi];
                if ((word >> lane) & 1u) {
                    const int pos = wpre[wi] + __popc(word & ((1u << lane) - 1u));
                    if (pos < kcap) out[pos] = j;
                }
            }
        }
        for (int i = total + tid; i < kcap; i += kSelThreads) out[i] = -1;
    }
    if (tid == 0) {
        nsel[(int64_t)b * c.hq + hq] = total;
        stamp_last(stamps, kStampSelect);
    }
}

template <int D, typename T>
static cudaError_t launch_score_t(const CacheView& c, const CUtensorMap& tstats, const void* q,
                                  double scale, int first_order, float* scores, int ld, float* gread,
                                  float* aw, KernelStamps* stamps, int32_t* status, cudaStream_t s) {
    using S = ScoreShape<D>;
    const int groups = c.batch * c.hkv;
    const int ntile = (c.mbp + kTile - 1) / kTile;
    const int64_t nitems = (int64_t)groups * (S::kReadoutParts + ntile);
    const int grid = (int)std::min<int64_t>((nitems + kScorePairs - 1) / kScorePairs,
                                            (int64_t)kScoreCtasPerSm * kNumSms);
    cudaError_t e = cudaFuncSetAttribute(score_kernel<D, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(score_kernel<D, T>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    return launch_pdl(score_kernel<D, T>, dim3(grid), dim3(kScoreWarps * 32), S::kSmem, s, tstats,
                      c, (const T*)q, scale, log((double)c.bs), first_order, scores, ld, gread, aw,
                      ntile, stamps, status);
}

int score_readout_parts(int d) {
    return d == 128 ? ScoreShape<128>::kReadoutParts : ScoreShape<64>::kReadoutParts;
}

cudaError_t launch_score(const CacheView& c, const CUtensorMap& tstats, int dtype, const void* q,
                         double scale, int first_order, float* scores, int ld, float* gread,
                         float* aw, KernelStamps* stamps, int32_t* status, cudaStream_t s) {
    if (dtype == SPLA_BF16)
        return c.d == 128 ? launch_score_t<128, __nv_bfloat16>(c, tstats, q, scale, first_order, scores, ld, gread, aw, stamps, status, s)
                          : launch_score_t<64, __nv_bfloat16>(c, tstats, q, scale, first_order, scores, ld, gread, aw, stamps, status, s);
    return c.d == 128 ? launch_score_t<128, float>(c, tstats, q, scale, first_order, scores, ld, gread, aw, stamps, status, s)
                      : launch_score_t<64, float>(c, tstats, q, scale, first_order, scores, ld, gread, aw, stamps, status, s);
}

template <int NT, int MAXB>
static cudaError_t launch_select_t(const CacheView& c, int top_k, int n_sink, int n_local,
                                   const float* scores, int ld, uint32_t* bits, int nw,
                                   int32_t* nsel, int32_t* sel_idx, int kcap,
                                   KernelStamps* stamps, cudaStream_t s) {
    const size_t smem = (size_t)((c.mbp + 31) / 32) * 32 * sizeof(uint32_t);
    // static plus dynamic shared memory may pass the 48 KiB default
    cudaError_t e = cudaFuncSetAttribute(select_kernel<NT, MAXB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(select_kernel<NT, MAXB>, dim3(c.batch * c.hq), dim3(NT), smem, s, c, top_k,
                      n_sink, n_local, scores, ld, bits, nw, nsel, sel_idx, kcap, stamps);
}

// Threads per head by the table's capacity: a thread covers at most 64 blocks.
cudaError_t launch_select(const CacheView& c, int top_k, int n_sink, int n_local,
                          const float* scores, int ld, uint32_t* bits, int nw, int32_t* nsel,
                          int32_t* sel_idx, int kcap, KernelStamps* stamps, cudaStream_t s) {
    if (c.mbp <= kSelLongBlocks)
        return launch_select_t<512, SPLA_MAX_BLOCKS_PER_SEQ>(c, top_k, n_sink, n_local, scores,
                                                             ld, bits, nw, nsel, sel_idx, kcap,
                                                             stamps, s);
    return launch_select_t<kSelThreadsLong, SPLA_MAX_BLOCKS_PER_SEQ>(
        c, top_k, n_sink, n_local, scores, ld, bits, nw, nsel, sel_idx, kcap, stamps, s);
}

}  // namespace spla
