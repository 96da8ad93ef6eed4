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
//   bc_phi_kernel      phi = exp(k - m*) of every token, once (the kept tokens'
//                      linear-attention weights become dot products with it);
//   bc_query_kernel    grid (max_len, batch*Hkv), one warp per query head of the
//                      group, lanes over dimensions (every statistics, K, V and
//                      phi row one coalesced load, dot products as warp sums):
//                      fp64 block scores over the complete earlier blocks,
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
    const float* phi;       // [batch*Hkv][max_len][d]: exp(k - m*) of every token
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

// ------------------------------------------------------------------ feature map
// phi[bh][t][i] = exp(k_t,i - m*_i) for every token (the query kernel's linear-
// attention weights are then dot products): one thread per 8 dimensions of a token.
__global__ void __launch_bounds__(256) bc_phi_kernel(CacheView c, const __nv_bfloat16* k_all,
                                                     int max_len, float* phi) {
    constexpr int d = kBcD;
    pdl_trigger();
    pdl_wait();
    const int bh = blockIdx.y, b = bh / c.hkv, h = bh % c.hkv;
    int32_t L = c.lens[b];
    L = max(0, min(L, max_len));
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // (t, 8-dim group)
    const int t = (int)(e / (d / 8)), g8 = (int)(e % (d / 8));
    if (t >= L) return;
    const uint4 q = *reinterpret_cast<const uint4*>(
        k_all + (((int64_t)b * max_len + t) * c.hkv + h) * d + 8 * g8);
    const __nv_bfloat16* kv = reinterpret_cast<const __nv_bfloat16*>(&q);
    const float* mr = c.m + (int64_t)bh * d + 8 * g8;
    float o[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) o[u] = expf(__bfloat162float(kv[u]) - mr[u]);
    float4* dst = reinterpret_cast<float4*>(phi + ((int64_t)bh * max_len + t) * d + 8 * g8);
    dst[0] = make_float4(o[0], o[1], o[2], o[3]);
    dst[1] = make_float4(o[4], o[5], o[6], o[7]);
}

// ------------------------------------------------------------------ queries
template <typename T>
__global__ void __launch_bounds__(kBcThreads, 4) bc_query_kernel(CacheView c, BcArgs a) {
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

    // ---- scores of the complete earlier blocks (fp64 dot products, fp32 log1p): warp w
    //      takes blocks w, w + 4, ...; lane l reads dimensions [4l, 4l + 4) of the
    //      block's mean and variance (one coalesced load each) for every head
    {
        const double lgB = log((double)bs);
        const int nwarps = kBcThreads / 32;
        for (int j = warp; j < J; j += nwarps) {
            const float* st = c.stats + (((int64_t)b * c.hkv + h) * c.mbp + j) * 2 * d + 4 * lane;
            const float4 mu = *reinterpret_cast<const float4*>(st);
            const float4 va = *reinterpret_cast<const float4*>(st + d);
            const float mv[4] = {mu.x, mu.y, mu.z, mu.w};
            const float vv[4] = {va.x, va.y, va.z, va.w};
            for (int g = 0; g < G; ++g) {
                double m1 = 0.0, m2 = 0.0;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const double qi = (double)qv[g][4 * lane + e] * a.scale;
                    m1 = fma((double)mv[e], qi, m1);
                    m2 = fma((double)vv[e], qi * qi, m2);
                }
#pragma unroll
                for (int o = 16; o; o >>= 1) {
                    m1 += __shfl_xor_sync(0xffffffffu, m1, o);
                    m2 += __shfl_xor_sync(0xffffffffu, m2, o);
                }
                if (lane == 0) {
                    double sv = lgB + m1;
                    if (!a.first_order) sv += (double)log1pf((float)(0.5 * m2));
                    sc[g * js + j] = (float)sv;
                }
            }
        }
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
    //      the kept complete blocks' linear-attention terms on the same tokens. Lane l
    //      owns dimensions [4l, 4l + 4): every token's K, V and phi rows are read by the
    //      whole warp in one coalesced load each; the two dot products (q.k, a.phi(k))
    //      are warp sums; four tokens' loads are in flight together.
    const T* kp = static_cast<const T*>(c.k_pool);
    const T* vp = static_cast<const T*>(c.v_pool);
    const float sl2 = (float)(a.scale * 1.4426950408889634);
    float qd[4], ad[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) { qd[e] = qv[g][4 * lane + e]; ad[e] = aw[g][4 * lane + e]; }
    float mrun = -SPLA_INF, lsum = 0.f, acc[4], ntl[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) { acc[e] = 0.f; ntl[e] = 0.f; }
    float dtl = 0.f;
    int kept_complete = 0;
    constexpr int U = 4;                         // tokens per step
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
        const T* kbk = kp + ((int64_t)phys * c.hkv + h) * bs * d + 4 * lane;
        const T* vbk = vp + ((int64_t)phys * c.hkv + h) * bs * d + 4 * lane;
        const float* pbk = a.phi + ((int64_t)bh * a.max_len + (int64_t)j * bs) * d + 4 * lane;
        for (int u0 = 0; u0 < ntok; u0 += U) {
            float kx[U][4], vx[U][4], fx[U][4];
#pragma unroll
            for (int r = 0; r < U; ++r) {
                const int u = u0 + r;
#pragma unroll
                for (int e = 0; e < 4; ++e) kx[r][e] = vx[r][e] = fx[r][e] = 0.f;
                if (u < ntok) {
                    const uint2 k2 = *reinterpret_cast<const uint2*>(kbk + (int64_t)u * d);
                    const uint2 v2 = *reinterpret_cast<const uint2*>(vbk + (int64_t)u * d);
                    kx[r][0] = bf16_lo(k2.x); kx[r][1] = bf16_hi(k2.x);
                    kx[r][2] = bf16_lo(k2.y); kx[r][3] = bf16_hi(k2.y);
                    vx[r][0] = bf16_lo(v2.x); vx[r][1] = bf16_hi(v2.x);
                    vx[r][2] = bf16_lo(v2.y); vx[r][3] = bf16_hi(v2.y);
                    if (!cur) {
                        const float4 f = *reinterpret_cast<const float4*>(pbk + (int64_t)u * d);
                        fx[r][0] = f.x; fx[r][1] = f.y; fx[r][2] = f.z; fx[r][3] = f.w;
                    }
                }
            }
            float lg[U], wv[U];
#pragma unroll
            for (int r = 0; r < U; ++r) {
                float dp = 0.f, wp = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    dp = fmaf(qd[e], kx[r][e], dp);
                    wp = fmaf(ad[e], fx[r][e], wp);
                }
                lg[r] = dp;
                wv[r] = wp;
            }
#pragma unroll
            for (int o = 16; o; o >>= 1)
#pragma unroll
                for (int r = 0; r < U; ++r) {
                    lg[r] += __shfl_xor_sync(0xffffffffu, lg[r], o);
                    wv[r] += __shfl_xor_sync(0xffffffffu, wv[r], o);
                }
#pragma unroll
            for (int r = 0; r < U; ++r) {
                if (u0 + r >= ntok) continue;
                const float l2 = lg[r] * sl2;
                const float mnew = fmaxf(mrun, l2);
                const float f = (mrun == -SPLA_INF) ? 0.f : ex2(mrun - mnew);
                const float pw = ex2(l2 - mnew);
                lsum = fmaf(lsum, f, pw);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc[e] = fmaf(acc[e], f, pw * vx[r][e]);
                    if (!cur) ntl[e] = fmaf(wv[r], vx[r][e], ntl[e]);
                }
                if (!cur) dtl += wv[r];
                mrun = mnew;
            }
        }
    }
    // ---- the residual: the state before block J minus the kept complete blocks
    const float* Pj = a.P + ((int64_t)bh * a.nbp + J) * d * d + 4 * lane;
    const float* zj = a.zP + ((int64_t)bh * a.nbp + J) * d;
    double N[4], D = 0.0;
#pragma unroll
    for (int e = 0; e < 4; ++e) N[e] = 0.0;
#pragma unroll 4
    for (int i = 0; i < d; ++i) {
        const float ai = aw[g][i];
        const float4 pr = *reinterpret_cast<const float4*>(Pj + (int64_t)i * d);
        N[0] += (double)(ai * pr.x);
        N[1] += (double)(ai * pr.y);
        N[2] += (double)(ai * pr.z);
        N[3] += (double)(ai * pr.w);
    }
    {
        double zs = 0.0;
#pragma unroll
        for (int e = 0; e < 4; ++e) zs += (double)(ad[e] * zj[4 * lane + e]);
#pragma unroll
        for (int o = 16; o; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
        D = zs;
    }
    const double Dr = D - (double)dtl;
    const bool off = a.no_rla || kept_complete >= J;
    const bool unresolved = !off && !(Dr > 0.0);
    if (unresolved && lane == 0) set_status(a.status, SPLA_DEV_RLA_UNRESOLVED);
    float osp[4], orl[4], sq = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        osp[e] = lsum > 0.f ? acc[e] / lsum : 0.f;
        orl[e] = (off || unresolved) ? 0.f : (float)((N[e] - (double)ntl[e]) / Dr);
        sq = fmaf(orl[e], orl[e], sq);
    }
    sq = warp_sum(sq);
    const float inv = rsqrtf(sq / d + a.eps);
    const int64_t o0 = (((int64_t)b * a.max_len + t) * c.hq + hq) * d + 4 * lane;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float gm = a.gamma ? a.gamma[(int64_t)hq * d + 4 * lane + e] : 1.f;
        static_cast<T*>(a.out)[o0 + e] = from_f<T>(osp[e] + gm * orl[e] * inv);
        if (a.o_sp) a.o_sp[o0 + e] = osp[e];
        if (a.o_rl) a.o_rl[o0 + e] = orl[e];
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
    const size_t phi = groups * (size_t)max_len * kBcD * sizeof(float);
    auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
    return a256(rec) + a256(P) + a256(zP) + a256(phi);
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
    float* phi = zP + a256(groups * (splits + 1) * (size_t)kBcD * 4) / 4;
    cudaError_t e = launch_block_states(c, tk, tv, k_all, c.lens, max_len, rec, a.status, s);
    if (e != cudaSuccess) return e;
    e = launch_pdl(bc_prefix_kernel, dim3(kBcD / 8, c.batch * c.hkv), dim3(256), 0, s, c,
                   (const float*)rec, splits, P, zP, splits + 1);
    if (e != cudaSuccess) return e;
    e = launch_pdl(bc_phi_kernel, dim3((unsigned)(((int64_t)max_len * (kBcD / 8) + 255) / 256),
                                       c.batch * c.hkv),
                   dim3(256), 0, s, c, (const __nv_bfloat16*)k_all, (int)max_len, phi);
    if (e != cudaSuccess) return e;
    a.P = P;
    a.zP = zP;
    a.phi = phi;
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
