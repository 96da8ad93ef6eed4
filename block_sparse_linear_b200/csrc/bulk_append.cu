// a0, many tokens at once -- the global linear-attention state over a chunk of
// new tokens as a dense contraction on the tensor cores (SPLA technical summary,
// gist.science: section 2.2 for the state that linear attention over all blocks
// reads, section 2.3 for the feature map exp). For one (sequence, KV head) and
// new tokens t with keys k_t and values v_t:
//   m_new = max(m, max_t k_t)                            (per dimension i)
//   S[i][j] <- S[i][j] e^{m_i - m_new,i} + sum_t e^{k_t,i - m_new,i} v_t,j
//   z[i]    <- z[i] e^{m_i - m_new,i}    + sum_t e^{k_t,i - m_new,i}
// The sum over t is Phi^T V with Phi[t][i] = e^{k_t,i - m_c,i}: an M = d by N = d
// product over K = tokens, run on tcgen05 with the accumulator in tensor memory.
//
// Launches (the block kernel, which writes the tokens into the pool and recomputes
// the touched blocks' statistics, runs beside the first):
//   bulk_state_kernel  grid (splits, batch*Hkv), 320 threads: split c of a
//                      (sequence, KV head) takes new tokens [c*T, (c+1)*T), finds
//                      their per-dimension maximum m_c, and writes the partial
//                      state S_c = sum e^{k - m_c} v^T, z_c and m_c to the
//                      workspace;
//   bulk_merge_kernel  grid (d/8, batch*Hkv): m_new = max(m, max_c m_c), then the
//                      old state and every partial rescaled to m_new and added in
//                      split order (the result does not depend on timing).
//
// bulk_state_kernel roles: warp 0 issues the TMA loads (64-token tiles of K and V,
// two 64-dimension boxes each, 128-byte swizzle, no multicast) into a two-stage
// ring; warp 1 owns the tensor memory and issues the MMAs; warps 2..9 turn each
// K tile into Phi in place. Phi is split into three bf16 parts (hi + mid + lo
// carries 24 bits of its fp32 value, so the products lose nothing a fp32
// accumulation keeps); V is bf16 already and is used as loaded. Both operands
// stay in the layout TMA wrote: token rows of 128 bytes, i.e. M- and N-major
// tiles for the MMA (A = Phi^T is M x K with M contiguous, B = V is K x N with N
// contiguous). Each stage runs 3 parts x 4 k-steps of M128 N128 K16 MMAs into
// one 128 x 128 fp32 accumulator (128 TMEM columns).
#include "common.cuh"

namespace spla {

constexpr int kBulkTok = 64;                 // tokens per stage
constexpr int kBulkStages = 2;
constexpr int kBulkTile = 16384;             // 64 tokens x 128 dims bf16 (two 8 KiB boxes)
constexpr int kBulkStage = 4 * kBulkTile;    // Phi hi (in place of K), mid, lo, V
constexpr int kBulkXformWarps = 8;
constexpr int kBulkXform = 32 * kBulkXformWarps;
constexpr int kBulkThreads = 64 + kBulkXform;
constexpr int kBulkD = 128;
constexpr size_t kBulkSmem = (size_t)kBulkStages * kBulkStage + 1024;   // + alignment slack

// ------------------------------------------------------------------ tcgen05 plumbing
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: 128-byte swizzle, MN-major operand whose
// 64-element (128-byte) MN atoms lie lbo bytes apart and whose 8-row K groups lie
// sbo bytes apart; version field 1 (sm_100), base offset 0 (atoms 1024-aligned).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;
    d |= 2ull << 61;
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// MN-major, N = 128, M = 128.
constexpr uint32_t kBulkIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                ((uint32_t)(kBulkD >> 3) << 17) | ((uint32_t)(kBulkD >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// Arrives once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_u32(bar)) : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr) : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int u = 0; u < 32; ++u) v[u] = __uint_as_float(r[u]);
}

// 3-D tiled TMA load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int32_t x,
                                            int32_t y, int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        :: "r"(smem_u32(dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// Partial record of one split: S_c [d][d], then z_c [d], then m_c [d] (fp32).
__host__ __device__ constexpr int64_t bulk_record_floats(int d) { return (int64_t)d * d + 2 * d; }

__device__ __forceinline__ int bulk_count(const int32_t* n_new, int32_t max_new, int b) {
    const int32_t n = n_new[b];
    return n < 0 ? 0 : (n > max_new ? max_new : n);
}

// The input views tk, tv are [batch*max_new rows][Hkv][d] bf16 with boxes of 64
// dimensions x 1 head x 64 tokens.
__global__ void __launch_bounds__(kBulkThreads, 1)
bulk_state_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                  const __nv_bfloat16* __restrict__ k_new, const int32_t* __restrict__ n_new,
                  int32_t max_new, int hkv, int tsplit, float* __restrict__ part,
                  int32_t* status) {
    extern __shared__ unsigned char bulk_smem_raw[];
    __shared__ __align__(8) uint64_t full[kBulkStages], ready[kBulkStages], empty[kBulkStages];
    __shared__ __align__(8) uint64_t done;
    __shared__ uint32_t tmem_base_sh;
    __shared__ float red[kBulkXform / 16][kBulkD];  // per-thread-row partial max / z
    __shared__ float mloc[kBulkD];

    // stage buffers on 1024-byte boundaries of the shared window (the swizzle atom)
    unsigned char* smem = bulk_smem_raw + ((1024u - (smem_u32(bulk_smem_raw) & 1023u)) & 1023u);
    const int split = blockIdx.x, bh = blockIdx.y;
    const int b = bh / hkv, h = bh % hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int n = bulk_count(n_new, max_new, b);
    const int t0 = split * tsplit;
    const int ntok = max(0, min(n, t0 + tsplit) - t0);
    // everything earlier on the stream (the previous call's merge reads this workspace,
    // its length advance is what the block kernel after this one reads) is complete
    // before this kernel lets the block kernel launch
    pdl_wait();
    pdl_trigger();
    if (ntok == 0) return;                          // no partial: the merge skips this split
    const int ntiles = (ntok + kBulkTok - 1) / kBulkTok;
    const int row0 = b * max_new + t0;              // first input row of this split

    if (threadIdx.x == 0) {
        for (int s = 0; s < kBulkStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&ready[s], kBulkXformWarps);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&done, 1);
        fence_barrier_init();
        prefetch_tmap(&tk);
        prefetch_tmap(&tv);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(&tmem_base_sh)), "r"(kBulkD) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            int it = 0;
            for (; it < ntiles; ++it) {
                const int s = it % kBulkStages;
                if (it >= kBulkStages &&
                    !mbar_wait_bounded(&empty[s], ((it / kBulkStages) - 1) & 1)) {
                    set_status(status, SPLA_DEV_TIMEOUT);
                    break;
                }
                unsigned char* st = smem + s * kBulkStage;
                mbar_arrive_expect_tx(&full[s], 4 * 8192);
                const int z = row0 + it * kBulkTok;
                tma_load_3d(st, &tk, &full[s], 0, h, z);
                tma_load_3d(st + 8192, &tk, &full[s], 64, h, z);
                tma_load_3d(st + 3 * kBulkTile, &tv, &full[s], 0, h, z);
                tma_load_3d(st + 3 * kBulkTile + 8192, &tv, &full[s], 64, h, z);
            }
            // the last copies issued into each slot have landed before the CTA may leave
            for (int j = max(0, it - kBulkStages); j < it; ++j)
                mbar_wait_bounded(&full[j % kBulkStages], (j / kBulkStages) & 1);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t base = smem_u32(smem);
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % kBulkStages;
                if (!mbar_wait_bounded(&ready[s], (it / kBulkStages) & 1)) {
                    set_status(status, SPLA_DEV_TIMEOUT);
                    break;
                }
                tc_fence_after();
                const uint32_t st = base + s * kBulkStage;
#pragma unroll
                for (int p = 0; p < 3; ++p)
#pragma unroll
                    for (int kk = 0; kk < kBulkTok / 16; ++kk) {
                        const uint64_t ad = umma_desc_sw128(st + p * kBulkTile + kk * 2048, 8192, 1024);
                        const uint64_t bd = umma_desc_sw128(st + 3 * kBulkTile + kk * 2048, 8192, 1024);
                        umma_bf16(tmem, ad, bd, kBulkIdesc, (it | p | kk) != 0);
                    }
                umma_commit(&empty[s]);             // frees the stage once these MMAs are done
            }
            umma_commit(&done);
            // no MMA of this CTA is in flight once `done` has fired
            if (!mbar_wait_bounded(&done, 0)) set_status(status, SPLA_DEV_TIMEOUT);
        }
    } else {
        // ---------------------------------------------------------- Phi producers + epilogue
        const int x = threadIdx.x - 64;             // 0 .. 255
        const int g = x & 15;                       // dimension group: dims 8g .. 8g+7
        const int r0 = x >> 4;                      // token rows r0 + 16u
        // pass 1: per-dimension maximum of this split's keys (read straight from global)
        float mx[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[e] = -SPLA_INF;
        // eight loads in flight per thread before any of them is used
        for (int t = r0; t < ntok; t += 16 * 8) {
            uint4 q[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (t + 16 * u < ntok)
                    q[u] = *reinterpret_cast<const uint4*>(
                        k_new + (((int64_t)(row0 + t + 16 * u)) * hkv + h) * kBulkD + 8 * g);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (t + 16 * u < ntok) {
                    const __nv_bfloat16* e8 = reinterpret_cast<const __nv_bfloat16*>(&q[u]);
#pragma unroll
                    for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], __bfloat162float(e8[e]));
                }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) red[r0][8 * g + e] = mx[e];
        asm volatile("bar.sync 1, %0;" :: "n"(kBulkXform));
        if (x < kBulkD) {
            float m = red[0][x];
            for (int r = 1; r < kBulkXform / 16; ++r) m = fmaxf(m, red[r][x]);
            mloc[x] = m;
        }
        asm volatile("bar.sync 1, %0;" :: "n"(kBulkXform));
        float mk[8], zacc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            mk[e] = mloc[8 * g + e];
            zacc[e] = 0.f;
        }
        // pass 2: Phi tiles. Thread x owns, in every stage, the 16-byte chunk of
        // dimensions 8g..8g+7 in rows r0 + 16u; under the 128-byte swizzle that
        // chunk sits at position (g % 8) ^ (row % 8) of its row, and row % 8 = r0 % 8.
        const int box = g >> 3;
        const int pos = (g & 7) ^ (r0 & 7);
        bool ok = true;
        for (int it = 0; it < ntiles; ++it) {
            const int s = it % kBulkStages;
            const bool got = mbar_wait_bounded(&full[s], (it / kBulkStages) & 1);
            if (!__all_sync(0xffffffffu, got)) {
                if (lane == 0) set_status(status, SPLA_DEV_TIMEOUT);
                ok = false;
                break;
            }
            unsigned char* st = smem + s * kBulkStage;
#pragma unroll
            for (int u = 0; u < kBulkTok / 16; ++u) {
                const int r = r0 + 16 * u;
                const int off = box * 8192 + r * 128 + pos * 16;
                uint4* hi = reinterpret_cast<uint4*>(st + off);
                uint4* mid = reinterpret_cast<uint4*>(st + kBulkTile + off);
                uint4* lo = reinterpret_cast<uint4*>(st + 2 * kBulkTile + off);
                if (it * kBulkTok + r < ntok) {
                    const uint4 q = *hi;
                    const __nv_bfloat16* e8 = reinterpret_cast<const __nv_bfloat16*>(&q);
                    uint32_t ph[4], pm[4], pl[4];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        float f[2];
#pragma unroll
                        for (int w = 0; w < 2; ++w) {
                            f[w] = expf(__bfloat162float(e8[e + w]) - mk[e + w]);
                            zacc[e + w] += f[w];
                        }
                        const __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]);
                        const float r1x = f[0] - __low2float(a), r1y = f[1] - __high2float(a);
                        const __nv_bfloat162 bm = __floats2bfloat162_rn(r1x, r1y);
                        const __nv_bfloat162 c = __floats2bfloat162_rn(r1x - __low2float(bm),
                                                                       r1y - __high2float(bm));
                        ph[e / 2] = *reinterpret_cast<const uint32_t*>(&a);
                        pm[e / 2] = *reinterpret_cast<const uint32_t*>(&bm);
                        pl[e / 2] = *reinterpret_cast<const uint32_t*>(&c);
                    }
                    *hi = make_uint4(ph[0], ph[1], ph[2], ph[3]);
                    *mid = make_uint4(pm[0], pm[1], pm[2], pm[3]);
                    *lo = make_uint4(pl[0], pl[1], pl[2], pl[3]);
                } else {
                    // rows past this split's tokens: Phi = 0 and V = 0 (the input rows
                    // there belong to other tokens or hold anything)
                    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
                    *hi = zero;
                    *mid = zero;
                    *lo = zero;
                    *reinterpret_cast<uint4*>(st + 3 * kBulkTile + off) = zero;
                }
            }
            fence_proxy_async();                    // generic writes -> tensor-core reads
            __syncwarp();
            if (lane == 0) mbar_arrive(&ready[s]);
        }
        float* rec = part + ((int64_t)bh * gridDim.x + split) * bulk_record_floats(kBulkD);
        asm volatile("bar.sync 1, %0;" :: "n"(kBulkXform));
#pragma unroll
        for (int e = 0; e < 8; ++e) red[r0][8 * g + e] = zacc[e];
        asm volatile("bar.sync 1, %0;" :: "n"(kBulkXform));
        if (x < kBulkD) {
            float zs = 0.f;
            for (int r = 0; r < kBulkXform / 16; ++r) zs += red[r][x];
            rec[kBulkD * kBulkD + x] = zs;
            rec[kBulkD * kBulkD + kBulkD + x] = mloc[x];
        }
        // accumulator: warp w reads TMEM lanes 32 (w % 4) .. +31 (rows i of S_c);
        // the two warps of a lane quarter take columns [0, 64) and [64, 128)
        const bool all_ok = __all_sync(0xffffffffu, ok);
        const bool fired = all_ok && mbar_wait_bounded(&done, 0);
        if (__all_sync(0xffffffffu, fired)) {
            tc_fence_after();
            const int quarter = warp & 3;
            const int chalf = (warp - 2) >> 2;      // warps 2..5 -> 0, 6..9 -> 1
            const int i = 32 * quarter + lane;
            float* srow = rec + (int64_t)i * kBulkD;
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                const int col = 64 * chalf + 32 * cb;
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)col, v);
#pragma unroll
                for (int u = 0; u < 32; u += 4)
                    *reinterpret_cast<float4*>(srow + col + u) =
                        make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
            }
        } else if (lane == 0) {
            set_status(status, SPLA_DEV_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     :: "r"(tmem), "r"(kBulkD) : "memory");
    }
}

// Rows [8 rg, 8 rg + 8) of S (and of z, m) of one (sequence, KV head): warp r owns
// row 8 rg + r, lane l columns 4l .. 4l + 3. Partials are added in split order.
__global__ void __launch_bounds__(256)
bulk_merge_kernel(CacheView c, const int32_t* n_new, int32_t max_new, int splits, int tsplit,
                  const float* __restrict__ part) {
    pdl_trigger();
    pdl_wait();
    const int bh = blockIdx.y;
    const int b = bh / c.hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + warp;
    const int32_t L0 = c.lens[b], n = n_new[b];
    if (n <= 0 || n > max_new) return;             // flagged by the block kernel
    if (L0 < 0 || (int64_t)L0 + n > (int64_t)c.mbp * c.bs) return;
    constexpr int d = kBulkD;
    constexpr int64_t R = bulk_record_floats(d);
    const int nsp = min(splits, (n + tsplit - 1) / tsplit);
    const float* rec0 = part + (int64_t)bh * splits * R;
    const int64_t gidx = (int64_t)bh * d + row;
    const float m_old = c.m[gidx];
    float m_new = m_old;
    for (int sp = lane; sp < nsp; sp += 32) m_new = fmaxf(m_new, rec0[sp * R + d * d + d + row]);
    m_new = warp_max(m_new);
    const float f_old = (m_old == -SPLA_INF) ? 0.f : expf(m_old - m_new);
    float4* S4 = reinterpret_cast<float4*>(c.S + gidx * d) + lane;
    float4 acc = *S4;
    acc.x *= f_old; acc.y *= f_old; acc.z *= f_old; acc.w *= f_old;
    float zt = c.z[gidx] * f_old;
    constexpr int kBatch = 8;                       // partial rows in flight
    for (int sp0 = 0; sp0 < nsp; sp0 += kBatch) {
        float4 x[kBatch];
        float mc[kBatch], zc[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
            if (sp0 + u < nsp) {
                const float* rec = rec0 + (sp0 + u) * R;
                x[u] = reinterpret_cast<const float4*>(rec + (int64_t)row * d)[lane];
                mc[u] = rec[d * d + d + row];
                zc[u] = rec[d * d + row];
            }
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
            if (sp0 + u < nsp) {
                const float f = expf(mc[u] - m_new);
                acc.x = fmaf(x[u].x, f, acc.x);
                acc.y = fmaf(x[u].y, f, acc.y);
                acc.z = fmaf(x[u].z, f, acc.z);
                acc.w = fmaf(x[u].w, f, acc.w);
                zt = fmaf(zc[u], f, zt);
            }
    }
    *S4 = acc;
    if (lane == 0) {
        c.z[gidx] = zt;
        c.m[gidx] = m_new;
    }
}

// ------------------------------------------------------------------ host side
// Splits per (sequence, KV head): about one CTA per SM over the whole grid, each
// split a whole number of 64-token stages.
void bulk_shape(int batch, int hkv, int max_new, int* splits, int* tsplit) {
    const int groups = batch * hkv;
    int want = 148 / groups;
    if (want < 1) want = 1;
    const int stages = (max_new + kBulkTok - 1) / kBulkTok;
    int per = (stages + want - 1) / want;           // stages per split
    if (per < 1) per = 1;
    *tsplit = per * kBulkTok;
    *splits = (max_new + *tsplit - 1) / *tsplit;
    if (*splits < 1) *splits = 1;
}

size_t bulk_workspace_bytes(int batch, int hkv, int d, int max_new) {
    int splits, tsplit;
    bulk_shape(batch, hkv, max_new, &splits, &tsplit);
    return (size_t)batch * hkv * splits * bulk_record_floats(d) * sizeof(float);
}

cudaError_t launch_append_blocks(const CacheView& c, int dtype, const void* k_new,
                                 const void* v_new, const int32_t* n_new, int32_t max_new,
                                 int32_t* status, cudaStream_t s, bool with_rows, bool wait_last);
cudaError_t launch_append_advance(const CacheView& c, const int32_t* n_new, int32_t max_new,
                                  cudaStream_t s);

// Partial states of a whole sequence block by block (one split per block of B
// tokens): record (bh, j) holds S_j, z_j and m_j of block j's tokens. The inputs
// are the sequences' tokens from position 0.
cudaError_t launch_block_states(const CacheView& c, const CUtensorMap& tk, const CUtensorMap& tv,
                                const void* k_all, const int32_t* lens, int32_t max_len,
                                float* rec, int32_t* status, cudaStream_t s) {
    const int splits = (max_len + c.bs - 1) / c.bs;
    cudaError_t e = cudaFuncSetAttribute(bulk_state_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kBulkSmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(bulk_state_kernel, dim3(splits, c.batch * c.hkv), dim3(kBulkThreads),
                      kBulkSmem, s, tk, tv, (const __nv_bfloat16*)k_all, lens, max_len, c.hkv,
                      c.bs, rec, status);
}

// Order on the stream: state kernel (waits for everything before it, then lets the
// next launch in), block kernel (runs beside it on the SMs' remaining shared memory
// and registers; waits for the state kernel only at its end), merge, length advance.
cudaError_t launch_append_bulk(const CacheView& c, const CUtensorMap& tk, const CUtensorMap& tv,
                               const void* k_new, const void* v_new, const int32_t* n_new,
                               int32_t max_new, float* part, int32_t* status, cudaStream_t s) {
    int splits, tsplit;
    bulk_shape(c.batch, c.hkv, max_new, &splits, &tsplit);
    cudaError_t e = cudaFuncSetAttribute(bulk_state_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kBulkSmem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(bulk_state_kernel, dim3(splits, c.batch * c.hkv), dim3(kBulkThreads), kBulkSmem,
                   s, tk, tv, (const __nv_bfloat16*)k_new, n_new, max_new, c.hkv, tsplit, part,
                   status);
    if (e != cudaSuccess) return e;
    e = launch_append_blocks(c, SPLA_BF16, k_new, v_new, n_new, max_new, status, s,
                             /*with_rows=*/false, /*wait_last=*/true);
    if (e != cudaSuccess) return e;
    e = launch_pdl(bulk_merge_kernel, dim3(kBulkD / 8, c.batch * c.hkv), dim3(256), 0, s, c, n_new,
                   max_new, splits, tsplit, (const float*)part);
    if (e != cudaSuccess) return e;
    return launch_append_advance(c, n_new, max_new, s);
}

}  // namespace spla
