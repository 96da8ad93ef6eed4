// Block-causal form of the method over whole sequences (a prefill or training
// forward): query t sees tokens 0..t. Its own block J = t / B is attended exactly
// and causally; the complete earlier blocks 0..J-1 are the candidates, scored by
// the second-order Taylor estimate (SPLA technical summary, gist.science, section
// 2.1) and the top_k of them (after any sink blocks) attended exactly; the
// candidates left out are covered by linear attention (section 2.2), computed by
// subtraction from the state of the tokens before block J; out = o_sparse +
// gamma * RMSNorm(o_rla) (section 2.3).
//
// Launches (the cache already holds the sequences' tokens, their block
// statistics and the final state m):
//   bulk_state_kernel  with one split per block: S_j, z_j, m_j of every block
//                      (tensor cores, as for a bulk append);
//   bc_prefix_kernel   grid (d/8, batch*Hkv): P_J = sum_{j<J} S_j exp(m_j - m*),
//                      zP_J likewise, for J = 0 .. nb, m* the cache's final m
//                      (the running maximum over every token, an upper bound of
//                      every m_j); one warp per row of S, blocks in order;
//   bc_query_kernel    grid (max_len, batch*Hkv), one warp per query head of the
//                      group: fp64 block scores over the complete earlier blocks,
//                      the head's top_k by repeated warp arg-max over (score,
//                      lower block), exact online softmax over the kept blocks
//                      and the causal part of block J (K/V from the paged pool),
//                      the kept complete blocks' linear-attention terms N~, D~ on
//                      the same tokens, N, D from P_J, the subtraction in fp64,
//                      RMSNorm and the output.
#include "common.cuh"

namespace spla {

constexpr int kBcD = 128;
constexpr int kBcThreads = 128;                 // four warps: one per query head of a group
constexpr int kBcMaxBlocks = 4096;              // candidate blocks a query may score
constexpr int kBcMaxTopK = 256;

struct BcArgs {
    const void* q;          // [batch][max_len][Hq][d]
    void* out;              // [batch][max_len][Hq][d]
    float* o_sp;            // [batch][max_len][Hq][d] or null
    float* o_rl;            // same, or null
    const float* gamma;     // [Hq][d] or null
    const float* P;         // [batch*Hkv][nbp][d][d]
    const float* zP;        // [batch*Hkv][nbp][d]
    int32_t* status;
    int nbp;                // prefix states per group (blocks + 1)
    int jstride;            // floats per head in the shared score rows (>= blocks, multiple of 32)
    int max_len, top_k, n_sink, first_order, no_rla;
    double scale;
    float eps;
};

__host__ __device__ constexpr int64_t bc_record_floats(int d) { return (int64_t)d * d + 2 * d; }

// ------------------------------------------------------------------ prefix states
__global__ void __launch_bounds__(256) bc_prefix_kernel(CacheView c, const float* rec, int splits,
                                                        float* P, float* zP, int nbp) {
    constexpr int d = kBcD;
    constexpr int64_t R = bc_record_floats(d);
    pdl_trigger();
    pdl_wait();
    const int bh = blockIdx.y, b = bh / c.hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * 8 + warp;
    int32_t L = c.lens[b];
    L = max(0, min(L, c.mbp * c.bs));
    const int nbc = min(L / c.bs, splits);          // complete blocks
    const float mstar = c.m[(int64_t)bh * d + i];
    const float* rec0 = rec + (int64_t)bh * splits * R;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float zacc = 0.f;
    for (int J = 0; J <= nbc; ++J) {
        float4* dst = reinterpret_cast<float4*>(P + (((int64_t)bh * nbp + J) * d + i) * d) + lane;
        *dst = acc;
        if (lane == 0) zP[((int64_t)bh * nbp + J) * d + i] = zacc;
        if (J < nbc) {
            const float* r = rec0 + (int64_t)J * R;
            const float f = expf(r[d * d + d + i] - mstar);
            const float4 x = reinterpret_cast<const float4*>(r + (int64_t)i * d)[lane];
            acc.x = fmaf(x.x, f, acc.x);
            acc.y = fmaf(x.y, f, acc.y);
            acc.z = fmaf(x.z, f, acc.z);
            acc.w = fmaf(x.w, f, acc.w);
            zacc = fmaf(r[d * d + i], f, zacc);
        }
    }
}

// ------------------------------------------------------------------ queries
template <typename T>
__global__ void __launch_bounds__(kBcThreads) bc_query_kernel(CacheView c, BcArgs a) {
    constexpr int d = kBcD;
    constexpr int CPL = d / 32;                  // dimensions per lane
    extern __shared__ __align__(16) float smem_bc[];
    __shared__ __align__(16) float qv[4][d];     // the group's query rows
    __shared__ __align__(16) float aw[4][d];     // feature weights a_i of each head
    const int t = blockIdx.x, bh = blockIdx.y;
    const int b = bh / c.hkv, h = bh % c.hkv;
    const int G = c.group, bs = c.bs;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_wait();
    int32_t L = c.lens[b];
    L = max(0, min(L, c.mbp * bs));
    if (t >= L) return;
    const int J = t / bs;                        // candidates: blocks 0 .. J-1
    const int nwj = (J + 31) / 32;
    const int js = a.jstride;
    float* sc = smem_bc;                                              // [4][js] scores
    uint32_t* kept = reinterpret_cast<uint32_t*>(smem_bc + (size_t)4 * js);  // [4][js / 32]
    const T* qrow = static_cast<const T*>(a.q) + (((int64_t)b * a.max_len + t) * c.hq + h * G) * d;
    for (int e = tid; e < G * d; e += kBcThreads) qv[e / d][e % d] = to_f(qrow[e]);
    __syncthreads();

    // ---- scores of the complete earlier blocks (fp64 dot products, fp32 log1p)
    const double lgB = log((double)bs);
    for (int idx = tid; idx < G * J; idx += kBcThreads) {
        const int g = idx / J, j = idx % J;
        const float* st = c.stats + (((int64_t)b * c.hkv + h) * c.mbp + j) * 2 * d;
        double m1 = 0.0, m2 = 0.0;
        for (int i = 0; i < d; ++i) {
            const double qi = (double)qv[g][i] * a.scale;
            m1 = fma((double)st[i], qi, m1);
            m2 = fma((double)st[d + i], qi * qi, m2);
        }
        double s = lgB + m1;
        if (!a.first_order) s += (double)log1pf((float)(0.5 * m2));
        sc[g * js + j] = (float)s;
    }
    __syncthreads();

    // ---- selection: warp g keeps head g's sink blocks and top_k of the rest
    if (warp < G) {
        const int g = warp;
        uint32_t* kb = kept + g * (js / 32);
        for (int w = lane; w < nwj; w += 32) kb[w] = 0u;
        __syncwarp();
        const int fs = min(a.n_sink, J);
        const bool all = J - fs <= a.top_k;
        for (int j = lane; j < J; j += 32)
            if (all || j < fs) atomicOr(&kb[j >> 5], 1u << (j & 31));
        __syncwarp();
        if (!all) {
            for (int r = 0; r < a.top_k; ++r) {
                unsigned long long best = 0ull;
                for (int j = fs + lane; j < J; j += 32) {
                    if ((kb[j >> 5] >> (j & 31)) & 1u) continue;
                    const unsigned long long k =
                        ((unsigned long long)ordered_key(sc[g * js + j]) << 32) |
                        (uint32_t)~(uint32_t)j;
                    best = k > best ? k : best;
                }
#pragma unroll
                for (int o = 16; o; o >>= 1) {
                    const unsigned long long y = __shfl_xor_sync(0xffffffffu, best, o);
                    best = y > best ? y : best;
                }
                const int j = (int)~(uint32_t)best;
                if (best && lane == 0) kb[j >> 5] |= 1u << (j & 31);
                __syncwarp();
            }
        }
    }
    // every thread also needs m* for the feature weights
    const float* mrow = c.m + (int64_t)bh * d;
    if (warp < G) {
        const int g = warp;
        float x[CPL], mx = -SPLA_INF;
#pragma unroll
        for (int e = 0; e < CPL; ++e) {
            const int i = lane + 32 * e;
            x[e] = qv[g][i] + mrow[i];
            mx = fmaxf(mx, x[e]);
        }
        mx = warp_max(mx);
#pragma unroll
        for (int e = 0; e < CPL; ++e) aw[g][lane + 32 * e] = (mx == -SPLA_INF) ? 0.f : expf(x[e] - mx);
    }
    __syncthreads();
    if (warp >= G) return;
    const int g = warp, hq = h * G + g;
    const uint32_t* kb = kept + g * (js / 32);

    // ---- exact attention over the kept blocks and the causal part of block J, and
    //      the kept complete blocks' linear-attention terms on the same tokens
    const T* kp = static_cast<const T*>(c.k_pool);
    const T* vp = static_cast<const T*>(c.v_pool);
    const float sl2 = (float)(a.scale * 1.4426950408889634);
    float mrun = -SPLA_INF, lsum = 0.f, acc[CPL], ntl[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) { acc[e] = 0.f; ntl[e] = 0.f; }
    float dtl = 0.f;
    int kept_complete = 0;
    for (int j = 0; j <= J; ++j) {
        const bool cur = j == J;
        if (!cur && !((kb[j >> 5] >> (j & 31)) & 1u)) continue;
        if (!cur) ++kept_complete;
        const int32_t phys = c.table[(int64_t)b * c.mbp + j];
        if (phys < 0 || phys >= c.num_phys) {
            if (lane == 0) set_status(a.status, SPLA_DEV_BAD_BLOCK_TABLE);
            continue;
        }
        const int ntok = cur ? t - J * bs + 1 : bs;
        const T* kbk = kp + ((int64_t)phys * c.hkv + h) * bs * d;
        const T* vbk = vp + ((int64_t)phys * c.hkv + h) * bs * d;
        for (int u0 = 0; u0 < ntok; u0 += 32) {
            // lane u holds token u0 + u: its logit (log2 units) and its feature weight
            const int u = u0 + lane;
            float lg = -SPLA_INF, wt = 0.f;
            if (u < ntok) {
                const T* kr = kbk + (int64_t)u * d;
                float dot = 0.f, w = 0.f;
                for (int i = 0; i < d; ++i) {
                    const float kv = to_f(kr[i]);
                    dot = fmaf(qv[g][i], kv, dot);
                    if (!cur) w = fmaf(aw[g][i], expf(kv - mrow[i]), w);
                }
                lg = dot * sl2;
                wt = w;
            }
            const float mnew = fmaxf(mrun, warp_max(lg));
            const float f = (mrun == -SPLA_INF) ? 0.f : ex2(mrun - mnew);
            lsum *= f;
#pragma unroll
            for (int e = 0; e < CPL; ++e) acc[e] *= f;
            mrun = mnew;
            const int nu = min(32, ntok - u0);
            for (int x = 0; x < nu; ++x) {
                const float lgx = __shfl_sync(0xffffffffu, lg, x);
                const float wx = __shfl_sync(0xffffffffu, wt, x);
                const float p = ex2(lgx - mrun);
                lsum += p;
                const T* vr = vbk + (int64_t)(u0 + x) * d;
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    const float vv = to_f(vr[lane + 32 * e]);
                    acc[e] = fmaf(p, vv, acc[e]);
                    if (!cur) ntl[e] = fmaf(wx, vv, ntl[e]);
                }
                if (!cur) dtl += wx;
            }
        }
    }
    // ---- the residual: the state before block J minus the kept complete blocks
    const float* Pj = a.P + ((int64_t)bh * a.nbp + J) * d * d;
    const float* zj = a.zP + ((int64_t)bh * a.nbp + J) * d;
    double N[CPL], D = 0.0;
#pragma unroll
    for (int e = 0; e < CPL; ++e) N[e] = 0.0;
    for (int i = 0; i < d; ++i) {
        const float ai = aw[g][i];
#pragma unroll
        for (int e = 0; e < CPL; ++e) N[e] += (double)(ai * Pj[(int64_t)i * d + lane + 32 * e]);
    }
    {
        double zs = 0.0;
#pragma unroll
        for (int e = 0; e < CPL; ++e) zs += (double)(aw[g][lane + 32 * e] * zj[lane + 32 * e]);
#pragma unroll
        for (int o = 16; o; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
        D = zs;
    }
    const double Dr = D - (double)dtl;
    const bool off = a.no_rla || kept_complete >= J;
    const bool unresolved = !off && !(Dr > 0.0);
    if (unresolved && lane == 0) set_status(a.status, SPLA_DEV_RLA_UNRESOLVED);
    float osp[CPL], orl[CPL], sq = 0.f;
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
        osp[e] = lsum > 0.f ? acc[e] / lsum : 0.f;
        orl[e] = (off || unresolved) ? 0.f : (float)((N[e] - (double)ntl[e]) / Dr);
        sq = fmaf(orl[e], orl[e], sq);
    }
    sq = warp_sum(sq);
    const float inv = rsqrtf(sq / d + a.eps);
    const int64_t o0 = (((int64_t)b * a.max_len + t) * c.hq + hq) * d;
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
        const int i = lane + 32 * e;
        const float gm = a.gamma ? a.gamma[(int64_t)hq * d + i] : 1.f;
        static_cast<T*>(a.out)[o0 + i] = from_f<T>(osp[e] + gm * orl[e] * inv);
        if (a.o_sp) a.o_sp[o0 + i] = osp[e];
        if (a.o_rl) a.o_rl[o0 + i] = orl[e];
    }
}

// ------------------------------------------------------------------ host side
int bc_max_blocks() { return kBcMaxBlocks; }
int bc_max_top_k() { return kBcMaxTopK; }

size_t bc_workspace_bytes(int batch, int hkv, int bs, int max_len) {
    const int splits = (max_len + bs - 1) / bs;
    const size_t groups = (size_t)batch * hkv;
    const size_t rec = groups * splits * bc_record_floats(kBcD) * sizeof(float);
    const size_t P = groups * (splits + 1) * (size_t)kBcD * kBcD * sizeof(float);
    const size_t zP = groups * (splits + 1) * (size_t)kBcD * sizeof(float);
    auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
    return a256(rec) + a256(P) + a256(zP);
}

cudaError_t launch_block_states(const CacheView& c, const CUtensorMap& tk, const CUtensorMap& tv,
                                const void* k_all, const int32_t* lens, int32_t max_len,
                                float* rec, int32_t* status, cudaStream_t s);

cudaError_t launch_block_causal(const CacheView& c, const CUtensorMap& tk, const CUtensorMap& tv,
                                const void* k_all, int32_t max_len, BcArgs a, char* ws,
                                cudaStream_t s) {
    const int splits = (max_len + c.bs - 1) / c.bs;
    const size_t groups = (size_t)c.batch * c.hkv;
    auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
    float* rec = reinterpret_cast<float*>(ws);
    float* P = reinterpret_cast<float*>(ws + a256(groups * splits * bc_record_floats(kBcD) * 4));
    float* zP = P + a256(groups * (splits + 1) * (size_t)kBcD * kBcD * 4) / 4;
    cudaError_t e = launch_block_states(c, tk, tv, k_all, c.lens, max_len, rec, a.status, s);
    if (e != cudaSuccess) return e;
    e = launch_pdl(bc_prefix_kernel, dim3(kBcD / 8, c.batch * c.hkv), dim3(256), 0, s, c,
                   (const float*)rec, splits, P, zP, splits + 1);
    if (e != cudaSuccess) return e;
    a.P = P;
    a.zP = zP;
    a.nbp = splits + 1;
    a.jstride = (splits + 31) / 32 * 32;
    const size_t smem = (size_t)4 * a.jstride * sizeof(float) +
                        (size_t)4 * (a.jstride / 32) * sizeof(uint32_t);
    e = cudaFuncSetAttribute(bc_query_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(bc_query_kernel<__nv_bfloat16>, dim3(max_len, c.batch * c.hkv),
                      dim3(kBcThreads), smem, s, c, a);
}

cudaError_t launch_block_causal_entry(const CacheView& c, const CUtensorMap& tk,
                                      const CUtensorMap& tv, const void* k_all, int32_t max_len,
                                      const void* q_all, const float* gamma, void* out,
                                      float* o_sp, float* o_rl, int top_k, int n_sink,
                                      int first_order, int no_rla, double scale, float eps,
                                      char* ws, int32_t* status, cudaStream_t s) {
    BcArgs a = {};
    a.q = q_all;
    a.out = out;
    a.o_sp = o_sp;
    a.o_rl = o_rl;
    a.gamma = gamma;
    a.status = status;
    a.max_len = max_len;
    a.top_k = top_k;
    a.n_sink = n_sink;
    a.first_order = first_order;
    a.no_rla = no_rla;
    a.scale = scale;
    a.eps = eps;
    return launch_block_causal(c, tk, tv, k_all, max_len, a, ws, s);
}

}  // namespace spla
