// a0 -- appending tokens: write K/V into the paged pool, recompute the block
// statistics of every touched block, and update the global linear-attention
// state (SPLA technical summary, gist.science: section 2.1 for the per-block
// mean and diagonal variance, section 2.2 for the global state that linear
// attention over all blocks reads, section 2.3 for the feature map exp).
//
// Two launches, stream-ordered:
//   append_kernel    grid (touched blocks + d/8 row groups, batch*Hkv), two
//                    independent roles that both read the old context_lens:
//                    CTAs x < nsb write the tokens of logical block
//                    L0/B + x, then its mean and population variance in fp64
//                    (two-pass, keys staged in shared memory); the other CTAs
//                    own 8 rows of S (and of z, m): m <- max(m, k_new), rescale
//                    by exp(m_old - m_new), add exp(k - m_new) v^T and
//                    exp(k - m_new);
//   append_advance   one CTA: context_lens[b] += n_new[b].
#include "common.cuh"

namespace spla {

// Validation shared by the three kernels: the same answer in each.
__device__ __forceinline__ bool append_ok(const CacheView& c, const int32_t* n_new,
                                          int32_t max_new, int b, int32_t* L0, int32_t* n) {
    int32_t l0 = c.lens[b];
    int32_t nn = n_new[b];
    *L0 = l0;
    *n = nn;
    if (nn < 0 || nn > max_new) return false;
    if (l0 < 0 || (int64_t)l0 + nn > (int64_t)c.mbp * c.bs) return false;
    return true;
}

// Tokens and statistics of logical block L0/B + x of one (sequence, KV head).
template <typename T>
__device__ void append_block(const CacheView& c, const T* k_new, const T* v_new,
                             const int32_t* n_new, int32_t max_new, int32_t* status, int b, int h,
                             int x, float* ktile) {
    int32_t L0, n;
    if (!append_ok(c, n_new, max_new, b, &L0, &n)) {
        if (x == 0 && h == 0 && threadIdx.x == 0)
            set_status(status, (n < 0 || n > max_new) ? SPLA_DEV_BAD_COUNT : SPLA_DEV_CAPACITY);
        return;
    }
    if (n == 0) return;
    const int bs = c.bs, d = c.d;
    const int lb = L0 / bs + x;                     // logical block this CTA owns
    const int64_t blk_lo = (int64_t)lb * bs;
    if (blk_lo >= (int64_t)L0 + n) return;
    const int32_t phys = c.table[(int64_t)b * c.mbp + lb];
    if (phys < 0 || phys >= c.num_phys) {
        if (threadIdx.x == 0) set_status(status, SPLA_DEV_BAD_BLOCK_TABLE);
        return;
    }
    const int t_beg = (int)(blk_lo > L0 ? blk_lo : (int64_t)L0);
    const int t_end = (int)((int64_t)L0 + n < blk_lo + bs ? (int64_t)L0 + n : blk_lo + bs);
    T* kp = (T*)c.k_pool + ((int64_t)phys * c.hkv + h) * bs * d;
    T* vp = (T*)c.v_pool + ((int64_t)phys * c.hkv + h) * bs * d;
    // write the new tokens of this block: 16-byte vectors when every buffer allows them
    const bool vec = ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new) |
                       reinterpret_cast<uintptr_t>(c.k_pool) |
                       reinterpret_cast<uintptr_t>(c.v_pool)) & 15) == 0;
    if (vec) {
        constexpr int EPV = 16 / sizeof(T);
        const int vpr = d / EPV;                     // vectors per token row
        const int nv = (t_end - t_beg) * vpr;
        // four K and four V vectors per thread in flight before any store
        constexpr int kCopyBatch = 4;
        for (int e0 = threadIdx.x; e0 < nv; e0 += kCopyBatch * blockDim.x) {
            int4 kx[kCopyBatch], vx[kCopyBatch];
#pragma unroll
            for (int r = 0; r < kCopyBatch; ++r) {
                const int e = e0 + r * blockDim.x;
                if (e < nv) {
                    const int t = t_beg + e / vpr, u = e % vpr;
                    const int64_t src = (((int64_t)b * max_new + (t - L0)) * c.hkv + h) * d + u * EPV;
                    kx[r] = *reinterpret_cast<const int4*>(k_new + src);
                    vx[r] = *reinterpret_cast<const int4*>(v_new + src);
                }
            }
#pragma unroll
            for (int r = 0; r < kCopyBatch; ++r) {
                const int e = e0 + r * blockDim.x;
                if (e < nv) {
                    const int t = t_beg + e / vpr, u = e % vpr;
                    const int64_t dst = (int64_t)(t - blk_lo) * d + u * EPV;
                    *reinterpret_cast<int4*>(kp + dst) = kx[r];
                    *reinterpret_cast<int4*>(vp + dst) = vx[r];
                    const T* ke = reinterpret_cast<const T*>(&kx[r]);
#pragma unroll
                    for (int q = 0; q < EPV; ++q) ktile[dst + q] = to_f(ke[q]);   // for the statistics
                }
            }
        }
    } else {
        const int nw = (t_end - t_beg) * d;
        for (int e = threadIdx.x; e < nw; e += blockDim.x) {
            const int t = t_beg + e / d, i = e % d;
            const int64_t src = (((int64_t)b * max_new + (t - L0)) * c.hkv + h) * d + i;
            kp[(int64_t)(t - blk_lo) * d + i] = k_new[src];
            vp[(int64_t)(t - blk_lo) * d + i] = v_new[src];
        }
    }
    // statistics over all tokens now in the block: the keys staged in shared memory
    // (the new ones above when vectors were used, the older ones -- or all of them --
    // read back from the pool with coalesced loads), then two passes per dimension in fp64
    const int nj = t_end - (int)blk_lo;
    if (!vec) __syncthreads();                       // the scalar writes above, before reading back
    {
        // 16-byte loads, a batch of them in flight before any store (d is a multiple
        // of 64, so a block's nj*d keys split into whole vectors)
        constexpr int EPV = 16 / sizeof(T);
        const int nvec = (vec ? t_beg - (int)blk_lo : nj) * d / EPV;
        const int4* src = reinterpret_cast<const int4*>(kp);
        constexpr int kBatch = 4;
        for (int v0 = threadIdx.x; v0 < nvec; v0 += kBatch * blockDim.x) {
            int4 x[kBatch];
#pragma unroll
            for (int k = 0; k < kBatch; ++k)
                if (v0 + k * (int)blockDim.x < nvec) x[k] = src[v0 + k * blockDim.x];
#pragma unroll
            for (int k = 0; k < kBatch; ++k) {
                const int v = v0 + k * blockDim.x;
                if (v < nvec) {
                    const T* e = reinterpret_cast<const T*>(&x[k]);
#pragma unroll
                    for (int u = 0; u < EPV; ++u) ktile[v * EPV + u] = to_f(e[u]);
                }
            }
        }
    }
    __syncthreads();
    float* st = c.stats + (((int64_t)b * c.hkv + h) * c.mbp + lb) * 2 * d;
    const int parts = blockDim.x / d;                // threads per dimension (2 at d=128, 4 at 64)
    const int i = threadIdx.x % d, part = threadIdx.x / d;
    __shared__ double red[256];
    double s = 0.0;
    for (int t = part; t < nj; t += parts) s += (double)ktile[t * d + i];
    red[threadIdx.x] = s;
    __syncthreads();
    double tot = 0.0;
    for (int p = 0; p < parts; ++p) tot += red[p * d + i];
    const double mean = tot / nj;
    __syncthreads();
    double q = 0.0;
    for (int t = part; t < nj; t += parts) {
        const double x = (double)ktile[t * d + i] - mean;
        q += x * x;
    }
    red[threadIdx.x] = q;
    __syncthreads();
    if (part == 0) {
        double qt = 0.0;
        for (int p = 0; p < parts; ++p) qt += red[p * d + i];
        st[i] = (float)mean;
        st[d + i] = (float)(qt / nj);
    }
}

// Rows [8*rg, +8) of S (and the same entries of z, m) of one (sequence, KV head).
// Warp r owns row r; lane l owns columns l, l+32, ... of that row. The row's state
// (m, z, S) and the first new token's k and v do not depend on the length or the
// count: they are loaded together with them, so a one-token append takes one round
// trip before its arithmetic.
template <typename T>
__device__ void append_rows(const CacheView& c, const T* k_new, const T* v_new,
                            const int32_t* n_new, int32_t max_new, int b, int h, int rg) {
    const int d = c.d;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = rg * 8 + warp;
    if (row >= d) return;
    const int64_t gidx = ((int64_t)b * c.hkv + h) * d + row;
    float* Srow = c.S + gidx * d;
    auto kval = [&](int t) -> float {
        return to_f(k_new[(((int64_t)b * max_new + t) * c.hkv + h) * d + row]);
    };
    constexpr int CPL = 4;                         // columns per lane (d <= 128)
    // loads that need neither the length nor the count (max_new >= 1 here)
    float s_old[CPL], v0[CPL];
    const T* vr0 = v_new + (((int64_t)b * max_new) * c.hkv + h) * d;
#pragma unroll
    for (int u = 0; u < CPL; ++u) {
        const int j = lane + 32 * u;
        s_old[u] = (j < d) ? Srow[j] : 0.f;
        v0[u] = (j < d) ? to_f(vr0[j]) : 0.f;
    }
    const float m_old = c.m[gidx], z_old = c.z[gidx];
    const float k0 = kval(0);
    int32_t L0, n;
    if (!append_ok(c, n_new, max_new, b, &L0, &n) || n == 0) return;
    // running max of this dimension over the new tokens
    float mx = (lane == 0) ? k0 : -SPLA_INF;
    for (int t = lane; t < n; t += 32)
        if (t > 0) mx = fmaxf(mx, kval(t));
    mx = warp_max(mx);
    const float m_new = fmaxf(m_old, mx);
    const float f = (m_old == -SPLA_INF) ? 0.f : expf(m_old - m_new);
    float acc[CPL], tot[CPL];
#pragma unroll
    for (int u = 0; u < CPL; ++u) {
        tot[u] = s_old[u] * f;
        acc[u] = 0.f;
    }
    float zacc = 0.f, ztot = z_old * f;
    // new tokens, summed in chunks of 256 before joining the running total
    for (int t = 0; t < n; ++t) {
        const float e = expf((t == 0 ? k0 : kval(t)) - m_new);
        const T* vr = v_new + (((int64_t)b * max_new + t) * c.hkv + h) * d;
#pragma unroll
        for (int u = 0; u < CPL; ++u) {
            const int j = lane + 32 * u;
            if (j < d) acc[u] = fmaf(e, t == 0 ? v0[u] : to_f(vr[j]), acc[u]);
        }
        zacc += e;
        if ((t & 255) == 255) {
#pragma unroll
            for (int u = 0; u < CPL; ++u) { tot[u] += acc[u]; acc[u] = 0.f; }
            ztot += zacc;
            zacc = 0.f;
        }
    }
#pragma unroll
    for (int u = 0; u < CPL; ++u) {
        const int j = lane + 32 * u;
        if (j < d) Srow[j] = tot[u] + acc[u];
    }
    if (lane == 0) {
        c.z[gidx] = ztot + zacc;
        c.m[gidx] = m_new;
    }
}

// One launch for both roles: CTAs x < nsb take blocks, the rest take row groups.
template <typename T>
__global__ void __launch_bounds__(256, 4) append_kernel(CacheView c, const T* k_new, const T* v_new,
                                                     const int32_t* n_new, int32_t max_new,
                                                     int nsb, int wait_last, int32_t* status) {
    extern __shared__ float ktile[];                 // [B][d], block role only
    const int b = blockIdx.y / c.hkv;
    const int h = blockIdx.y % c.hkv;
    pdl_trigger();
    // wait_last: the kernel before this one already waited for everything this one
    // reads and let it launch only then; waiting at the end keeps the kernels after
    // this one ordered behind that predecessor too
    if (!wait_last) pdl_wait();
    if ((int)blockIdx.x < nsb)
        append_block<T>(c, k_new, v_new, n_new, max_new, status, b, h, blockIdx.x, ktile);
    else
        append_rows<T>(c, k_new, v_new, n_new, max_new, b, h, blockIdx.x - nsb);
    if (wait_last) pdl_wait();
}

__global__ void append_advance_kernel(CacheView c, const int32_t* n_new, int32_t max_new) {
    pdl_trigger();
    pdl_wait();
    for (int b = threadIdx.x; b < c.batch; b += blockDim.x) {
        int32_t L0, n;
        if (append_ok(c, n_new, max_new, b, &L0, &n)) c.lens[b] = L0 + n;
    }
}

__global__ void cache_init_kernel(CacheView c) {
    const int64_t nsz = (int64_t)c.batch * c.hkv * c.d;
    const int64_t ssz = nsz * c.d;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < ssz;
         i += (int64_t)gridDim.x * blockDim.x) {
        c.S[i] = 0.f;
        if (i < nsz) {
            c.z[i] = 0.f;
            c.m[i] = -SPLA_INF;
        }
        if (i < c.batch) c.lens[i] = 0;
    }
}

// ------------------------------------------------------------------ host launchers
cudaError_t launch_cache_init(const CacheView& c, cudaStream_t s) {
    cache_init_kernel<<<296, 256, 0, s>>>(c);
    return cudaGetLastError();
}

// The block role alone: tokens into the pool and the touched blocks' statistics.
cudaError_t launch_append_blocks(const CacheView& c, int dtype, const void* k_new,
                                 const void* v_new, const int32_t* n_new, int32_t max_new,
                                 int32_t* status, cudaStream_t s, bool with_rows,
                                 bool wait_last) {
    const int nsb = (max_new + c.bs - 1) / c.bs + 1;         // blocks a sequence's tokens can touch
    dim3 grid(nsb + (with_rows ? (c.d + 7) / 8 : 0), c.batch * c.hkv);
    const size_t smem = (size_t)c.bs * c.d * sizeof(float);
    cudaError_t e = dtype == SPLA_BF16
        ? cudaFuncSetAttribute(append_kernel<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
        : cudaFuncSetAttribute(append_kernel<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dtype == SPLA_BF16) {
        using B16 = __nv_bfloat16;
        return launch_pdl(append_kernel<B16>, grid, dim3(256), smem, s, c, (const B16*)k_new,
                          (const B16*)v_new, n_new, max_new, nsb, wait_last ? 1 : 0, status);
    }
    return launch_pdl(append_kernel<float>, grid, dim3(256), smem, s, c, (const float*)k_new,
                      (const float*)v_new, n_new, max_new, nsb, wait_last ? 1 : 0, status);
}

cudaError_t launch_append_advance(const CacheView& c, const int32_t* n_new, int32_t max_new,
                                  cudaStream_t s) {
    return launch_pdl(append_advance_kernel, dim3(1), dim3(128), 0, s, c, n_new, max_new);
}

cudaError_t launch_append(const CacheView& c, int dtype, const void* k_new, const void* v_new,
                          const int32_t* n_new, int32_t max_new, int32_t* status,
                          cudaStream_t s) {
    if (max_new > 0) {
        cudaError_t e = launch_append_blocks(c, dtype, k_new, v_new, n_new, max_new, status, s,
                                             /*with_rows=*/true, /*wait_last=*/false);
        if (e != cudaSuccess) return e;
    }
    return launch_append_advance(c, n_new, max_new, s);
}

}  // namespace spla
