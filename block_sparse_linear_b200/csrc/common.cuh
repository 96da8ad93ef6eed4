// Device helpers shared by the SPLA kernels (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "spla.h"

#define SPLA_INF __int_as_float(0x7f800000)
#define SPLA_LOG2E 1.4426950408889634f

// SMs of a B200; grids of persistent kernels are sized from it.
constexpr int kNumSms = 148;

namespace spla {

// ------------------------------------------------------------------ launch-time description
// Everything a kernel needs about the cache, passed by value.
struct CacheView {
    const void* k_pool;
    const void* v_pool;
    float* stats;            // [batch][Hkv][mbp][2][d], logical block order
    float* S;                // [batch][Hkv][d][d]
    float* z;                // [batch][Hkv][d]
    float* m;                // [batch][Hkv][d]
    const int32_t* table;    // [batch][mbp]
    int32_t* lens;           // [batch]
    int32_t batch, mbp, num_phys;
    int32_t hq, hkv, group, d, bs;
};

// Workspace carve-up of one decode call (byte offsets from the base pointer).
struct DecodeLayout {
    int32_t nsplit;          // decode CTAs per (sequence, KV head)
    int32_t nw;              // 32-bit words of a per-head selection bitset
    int32_t kcap;            // top_k + n_sink + n_local
    int32_t rec;             // floats per partial record
    int32_t readout_parts;   // row ranges of S the global readout is split into
    int32_t max_per;         // union blocks one decode CTA may receive
    int32_t ld;              // floats between two heads' score rows (mbp rounded up to 4)
    size_t off_scores, off_bits, off_nsel, off_part, off_gread, off_aw, total;
};

// Device timestamps of one decode call (measurement only), one slot per SM so that
// CTAs leaving together do not queue on one address: for each kernel of the chain
// and each SM, ~(first CTA past its dependency wait) and the last CTA's exit, in
// ns of %globaltimer, raised with atomicMax (so both start from zero). The host
// takes the extremes over the SMs.
struct KernelStamps {
    unsigned long long first_n, last;
};
constexpr int kStampSlots = 256;               // >= SMs of the device (148 on a B200)
enum { kStampScore = 0, kStampSelect = 1, kStampDecode = 2, kStampCombine = 3, kStampCount = 4 };
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ KernelStamps* stamp_slot(KernelStamps* s, int kernel) {
    uint32_t sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    return s + kernel * kStampSlots + (sm % kStampSlots);
}
__device__ __forceinline__ void stamp_first(KernelStamps* s, int kernel) {
    if (s) atomicMax(&stamp_slot(s, kernel)->first_n, ~global_ns());
}
__device__ __forceinline__ void stamp_last(KernelStamps* s, int kernel) {
    if (s) atomicMax(&stamp_slot(s, kernel)->last, global_ns());
}

// Per-call arguments of the decode kernels beyond the cache.
struct DecodeArgs {
    const void* q;
    const float* gamma;         // [Hq][d] or null
    void* out;                  // [batch][Hq][d], dtype
    float* o_sp;                // [batch][Hq][d] or null
    float* o_rl;                // [batch][Hq][d] or null
    const uint32_t* bits;       // [batch][Hq][nw] selection bitsets
    const int32_t* nsel;        // [batch][Hq]
    float* part;                // [batch*Hkv][nsplit][G][rec]
    const float* gread;         // [batch*Hkv][nrd][G][d+4]: readout parts, N (d) then D
    const float* aw;            // [batch*Hkv][d][4] phi weights a_g,i (written by the scoring kernel)
    KernelStamps* stamps;       // [kStampCount][kStampSlots] or null
    int32_t* status;
    int nw, nsplit, max_per, no_rla, nrd;
    float sl2, eps;
};

// Partial record of one decode CTA for one query head:
//   [0] m (running max, log2 units), [1] l (softmax denominator),
//   [2] D~_part, [3] unused, [4..4+d) acc, [4+d..4+2d) N~_part
// (the kept blocks' linear-attention numerator and denominator over this CTA's share)
__host__ __device__ inline int rec_floats(int d) { return 2 * d + 4; }

// ------------------------------------------------------------------ small math
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t ordered_key(float f) {
    // Monotone map float -> uint32 (larger float, larger key); 0 is below every float.
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x = lo (low 16 bits)
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Packed fp32 pair arithmetic (sm_100): one instruction for two lanes of work.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void set_status(int32_t* st, int32_t bits) {
    if (st) atomicOr(st, bits);
}

// ------------------------------------------------------------------ programmatic dependent launch
// Every kernel after the first of a call is launched with programmatic stream
// serialisation: it may start while its predecessor drains, and waits here
// before touching anything the predecessor (or an earlier kernel) wrote.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel in the stream launch once every CTA of this grid has run this.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ mbarrier / TMA (no multicast)
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait: returns false after `limit` unsuccessful polls.
constexpr uint32_t kWaitLimit = 1u << 22;
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// 2-D tiled TMA load into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        :: "r"(smem_u32(dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y) : "memory");
}

// L2 prefetch of one tile of a 2-D tensor map (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_2d(const void* tmap, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];"
                 :: "l"(tmap), "r"(x), "r"(y) : "memory");
}

// Bring a kernel-parameter tensor map into the TMA unit's descriptor cache.
__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" :: "l"(tmap) : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory (16-byte aligned, size a
// multiple of 16), completing on `bar`. No multicast.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// ------------------------------------------------------------------ warp-level MMA plumbing
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}
// D += A(16x16 bf16, row) * B(16x8 bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float* c, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled box
// (row pitch 128 B; chunk index XOR row mod 8), as TMA's 128B swizzle writes it.
__device__ __forceinline__ uint32_t swz128(int row, int chunk) {
    return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

#ifdef __CUDACC__
// Host: launch `kern` with programmatic stream serialisation.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
#endif

}  // namespace spla
