// nosa_common.cuh -- device helpers shared by the libnosa kernels (sm_100a).
//
// Inline-PTX wrappers for the Blackwell/Hopper asynchronous data path
// (mbarrier, TMA tiled loads, bulk copies), the bf16 tensor-core fragment
// instructions used by the decode kernel, and the fixed problem geometry.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nosa.h"

namespace nosa {

constexpr int kD = 128;                       // head dimension
constexpr int kBlock = 64;                    // tokens per block
constexpr int kSub = 16;                      // tokens per sub-block
constexpr int kSubPerBlock = kBlock / kSub;   // 4
constexpr int kRowBytes = kD * 2;             // one bf16 key or value row: 256 B
constexpr int kHalfBlockBytes = kBlock * kRowBytes;  // keys (or values) of a block: 16 KiB
constexpr int kBlockBytes = 2 * kHalfBlockBytes;     // keys + values of a block: 32 KiB
constexpr int kMaxG = 8;                      // query heads per kv head handled by one tile
constexpr int kMaxKq = 32;                    // Gamma_q fits one warp-wide sorted list
constexpr int kMaxKe = 256;
constexpr int kHeadH = NOSA_EVICT_HIDDEN;             // hidden width of the eviction head
constexpr long long kWaitCycles = 1ll << 32;  // ~2 s at 2 GHz: bound on every mbarrier wait

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n"
        " .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete; false if the bound
// (SM clock cycles) ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, long long limit = kWaitCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) return false;
    }
    return true;
}

// ---- TMA / bulk copies ------------------------------------------------------
// 2-D tiled tensor load into shared memory, completing on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// Linear bulk copy global -> shared (16-byte aligned addresses, size multiple of 16).
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- shared / global vector access -------------------------------------------
__device__ __forceinline__ uint4 lds128(const void *p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ float4 lds128f(const void *p) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

// 16-byte load that bypasses L1 (data written by other CTAs of this grid, or host memory).
__device__ __forceinline__ uint4 ldcg128(const void *p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ---- tensor-core fragments ------------------------------------------------------
// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate (row-major A, column-major B).
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4],
                                          const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Transpose an 8x8 bf16 matrix held one row-pair per lane (lane/4 = row).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// A 32-bit global load that stays where the program puts it (after the asm statements before it).
__device__ __forceinline__ int32_t ld_volatile_s32(const int32_t *ptr) {
    int32_t v;
    asm volatile("ld.volatile.global.s32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

// Hand-off counter between CTAs: an atomic add at gpu scope with acquire-release semantics.  Issued
// by one thread after a barrier of its CTA, it releases every write the CTA made before the barrier
// to the CTA that later acquires the counter (release is cumulative), and acquires the writes that
// the earlier arrivals released; a barrier after it extends that to the rest of the CTA.
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(void *ctr, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(ctr), "r"(v) : "memory");
    return old;
}

// Flags between CTAs of one grid: a release store that publishes what the storing thread (and,
// through a barrier or fence before it, its CTA) wrote, and the acquiring load that sees it.
__device__ __forceinline__ void st_release_gpu(int32_t *flag, int32_t v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(flag), "r"(v) : "memory");
}

__device__ __forceinline__ int32_t ld_acquire_gpu(const int32_t *flag) {
    int32_t v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    return v;
}

// Wait until *flag != 0, acquiring what its writer released; false if the bound (SM clock
// cycles) ran out.
__device__ __forceinline__ bool flag_wait(const int32_t *flag, long long limit = kWaitCycles) {
    if (ld_acquire_gpu(flag)) return true;
    const long long t0 = clock64();
    while (!ld_acquire_gpu(flag)) {
        if (clock64() - t0 > limit) return false;
        __nanosleep(32);
    }
    return true;
}

// Orders this thread's earlier generic-proxy view of global memory (e.g. data acquired from
// another CTA) before its later asynchronous-proxy accesses (TMA and bulk copies).
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Order-preserving map of a finite float onto uint32 (larger float -> larger integer).
__device__ __forceinline__ uint32_t float_order(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Selection key: higher score first, then lower block id.  0 means "no entry".
// A score of -0.0 is keyed as +0.0: the two are equal scores, so the tie must
// go to the lower block id (float_order alone would rank -0.0 below +0.0).
__device__ __forceinline__ uint64_t select_key(float score, int32_t blk) {
    if (__float_as_uint(score) == 0x80000000u) score = 0.0f;
    return (static_cast<uint64_t>(float_order(score)) << 32) |
           static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(blk));
}

__device__ __forceinline__ int32_t key_block(uint64_t key) {
    return static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(key & 0xFFFFFFFFull));
}

__device__ __forceinline__ uint64_t shfl64(uint64_t v, int src) {
    uint32_t lo = __shfl_sync(0xFFFFFFFFu, static_cast<uint32_t>(v), src);
    uint32_t hi = __shfl_sync(0xFFFFFFFFu, static_cast<uint32_t>(v >> 32), src);
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

__device__ __forceinline__ uint64_t shfl_up64(uint64_t v, int d) {
    uint32_t lo = __shfl_up_sync(0xFFFFFFFFu, static_cast<uint32_t>(v), d);
    uint32_t hi = __shfl_up_sync(0xFFFFFFFFu, static_cast<uint32_t>(v >> 32), d);
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Warp-wide sorted list of the 32 best keys (lane i holds rank i, descending).
// Insert x if it ranks among them; the 32nd entry falls off.
__device__ __forceinline__ void list_insert(uint64_t &list, uint64_t x, int lane) {
    unsigned better = __ballot_sync(0xFFFFFFFFu, list > x);
    int pos = __popc(better);
    uint64_t up = shfl_up64(list, 1);
    if (lane > pos) list = up;
    else if (lane == pos) list = x;
}

// Offer one candidate key per lane (0 = none) to the list.
__device__ __forceinline__ void list_offer(uint64_t &list, uint64_t cand, int lane) {
    uint64_t thr = shfl64(list, 31);
    unsigned m = __ballot_sync(0xFFFFFFFFu, cand > thr);
    while (m) {
        int src = __ffs(m) - 1;
        m &= m - 1;
        uint64_t x = shfl64(cand, src);
        list_insert(list, x, lane);
    }
}

__device__ __forceinline__ uint64_t shfl_xor64(uint64_t v, int m) {
    uint32_t lo = __shfl_xor_sync(0xFFFFFFFFu, static_cast<uint32_t>(v), m);
    uint32_t hi = __shfl_xor_sync(0xFFFFFFFFu, static_cast<uint32_t>(v >> 32), m);
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Merge another warp-wide sorted list (descending, lane i = rank i) into `list`,
// keeping the 32 best of both: the elementwise max of one list and the other
// reversed is a bitonic sequence holding the top 32 of the union; five
// half-cleaner stages sort it back into descending order.
__device__ __forceinline__ void list_merge(uint64_t &list, uint64_t other, int lane) {
    const uint64_t rev = shfl64(other, 31 - lane);
    uint64_t m = list > rev ? list : rev;
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        const uint64_t p = shfl_xor64(m, j);
        const bool lower = (lane & j) == 0;
        m = lower ? (m > p ? m : p) : (m < p ? m : p);
    }
    list = m;
}

// ---- pooled-key scoring -----------------------------------------------------------
// This lane's 4 dims of one pooled-key row in shared memory (fp32 rows of 512 B, bf16 of 256 B).
__device__ __forceinline__ float4 row4(const uint8_t *tile, int row, int lane, float *) {
    return lds128f(tile + row * (kD * 4) + lane * 16);
}
__device__ __forceinline__ float4 row4(const uint8_t *tile, int row, int lane, __nv_bfloat16 *) {
    uint2 w;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];"
                 : "=r"(w.x), "=r"(w.y)
                 : "r"(smem_u32(tile + row * (kD * 2) + lane * 8)));
    return make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
}

// One level of a transpose-reduction of per-lane row values v[0..2N): lanes exchange the half
// they do not keep (the upper half where lane bit o is set) and add.
template <int N, int R>
__device__ __forceinline__ void reduce_level(float (&v)[R], int lane, int o) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const float send = upper ? v[i] : v[i + N];
        const float keep = upper ? v[i + N] : v[i];
        v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
    }
}

// ---- programmatic dependent launch ---------------------------------------------
// Every kernel of the decode chain is launched with programmatic stream
// serialization and waits here before its first global access: the wait returns
// once the previous kernel on the stream has completed and its writes are
// visible, so ordering is unchanged while the launch and CTA setup overlap the
// previous kernel's tail.  Every CTA waits, so completion stays transitive.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Let the next kernel on the stream launch now (its CTAs then wait in pdl_wait).
// Used by kernels whose successor is small or short-waiting, never before a
// long-running kernel's successor could hold SM resources needed elsewhere.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void set_error(uint32_t *err, uint32_t bits) {
    if (err) atomicOr(err, bits);
}

}  // namespace nosa
