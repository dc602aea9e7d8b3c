// Device-side building blocks for sm_100a: mbarriers, bulk async copies, scoped
// atomics, bounded waits, storage-type conversions.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "kie_internal.h"

#define KIE_DEV __device__ __forceinline__

// ------------------------------------------------------------------ clocks, fences, barriers

KIE_DEV uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

KIE_DEV void named_bar_sync(int id, int count) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory"); }

KIE_DEV uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

KIE_DEV unsigned long long ld_acquire_gpu_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

KIE_DEV void red_release_gpu_add_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

KIE_DEV uint32_t ld_acquire_sys_u32(const volatile uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

KIE_DEV void st_release_sys_u32(volatile uint32_t *p, uint32_t v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

KIE_DEV unsigned ld_volatile_u32(const unsigned *p) { return *(const volatile unsigned *)p; }

KIE_DEV unsigned ld_acquire_gpu_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Index check of a global write (the diagnostic build with KIE_CHECK_BOUNDS, which stands in
// for a memory checker): false, with DERR_BOUNDS and `where` recorded in the error word, when
// the index is out of range; the caller then skips the write. The product build compiles it
// to true.
KIE_DEV bool in_bounds(bool ok, unsigned *err, unsigned where) {
#ifdef KIE_CHECK_BOUNDS
    if (!ok) atomicCAS(err, 0u, ((unsigned)DERR_BOUNDS << 8) | (where & 0xFFu));
    return ok;
#else
    (void)err;
    (void)where;
    return true;
#endif
}

// ------------------------------------------------------------------ completion-based publication
//
// A release (fence.release, red.release, fence.acq_rel) at GPU scope waits until every memory
// transaction in flight on the SM has completed, the weight stream's bulk copies included: with
// a producer warp keeping 3 x 64 KB copies in flight, a 148-CTA grid barrier with a release
// arrive takes about 12 us instead of 1.3 (an acquire poll costs about the same as a relaxed
// one). So values that other CTAs read after a barrier are published by completion instead:
// each is written with an atomic at GPU scope, which is performed in L2 (the point of
// coherence) and returns the old value; the writer folds the returned values into a token and
// waits for the token (pub_wait) before the barrier's relaxed arrive; readers poll the
// barrier with acquire loads and read the values through L2 (ld.cg). The arrive thus follows
// the values' completion in L2 without a fence.

KIE_DEV void pub_u32(void *p, uint32_t v, uint32_t &tok) {
    uint32_t old;
    asm volatile("atom.relaxed.gpu.global.exch.b32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    tok ^= old;
}
KIE_DEV void pub_f32(float *p, float v, uint32_t &tok) { pub_u32(p, __float_as_uint(v), tok); }
KIE_DEV void pub_u64(void *p, unsigned long long v, uint32_t &tok) {
    unsigned long long old;
    asm volatile("atom.relaxed.gpu.global.exch.b64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
    tok ^= (uint32_t)old ^ (uint32_t)(old >> 32);
}
KIE_DEV void pub_f32x2(float *p, float a, float b, uint32_t &tok) {  // p 8-byte aligned
    pub_u64(p, (unsigned long long)__float_as_uint(a) | ((unsigned long long)__float_as_uint(b) << 32), tok);
}
KIE_DEV void pub_add_f32(float *p, float v, uint32_t &tok) {
    float old;
    asm volatile("atom.relaxed.gpu.global.add.f32 %0, [%1], %2;" : "=f"(old) : "l"(p), "f"(v) : "memory");
    tok ^= __float_as_uint(old);
}
// Waits until every value folded into `tok` has returned (the comparison needs them all); the
// store never happens in practice, and writes only a scratch word if it does.
KIE_DEV void pub_wait(uint32_t tok, volatile uint32_t *sink) {
    if (tok == 0x9E3779B9u) *sink = tok;
    asm volatile("" ::: "memory");
}

KIE_DEV void red_relaxed_gpu_add_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
KIE_DEV void red_relaxed_gpu_add_u32(unsigned *p, unsigned v) {
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Records the first device error (code, where). Later errors keep the first.
KIE_DEV void set_error(unsigned *err, unsigned code, unsigned where) {
    atomicCAS(err, 0u, (code << 8) | (where & 0xFFu));
}

// ------------------------------------------------------------------ mbarrier

KIE_DEV void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

KIE_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

KIE_DEV void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

// `count` arrivals at once
KIE_DEV void mbar_arrive_n(uint64_t *bar, uint32_t count) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
                 "r"(count)
                 : "memory");
}

KIE_DEV void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// Non-blocking test of an mbarrier phase (returns at once).
KIE_DEV bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Blocking test with a bound: the thread is suspended in hardware until the phase completes or
// about `ns` nanoseconds have passed, whichever comes first.
KIE_DEV bool mbar_try_wait_ns(uint64_t *bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Potentially blocking test: the thread may be suspended in hardware (up to the 1 ms hint)
// until the phase completes.
KIE_DEV bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase. Returns false on timeout or when *abort becomes set.
KIE_DEV bool mbar_wait(uint64_t *bar, uint32_t parity, long long timeout_ns, const volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (abort && *abort) return false;
        if ((long long)(globaltimer() - t0) > timeout_ns) return false;
    }
}

// ------------------------------------------------------------------ bulk async copy (TMA, 1-D, no multicast)

// Global -> this CTA's shared memory; completion is signalled as transaction bytes on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
KIE_DEV void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Reads 16 bytes at src into shared memory at dst asynchronously, with the 128-byte L2 fetch
// size: the line lands in L2 and stays there for a later bulk copy (on B200 the L2 prefetch
// instructions leave much of the data out of L2). The caller never reads dst; it waits for
// these copies (cp_async_wait_all) before its shared memory goes away.
KIE_DEV void l2_warm_line(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global.L2::128B [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
KIE_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Hint: bring the line holding p into this SM's L1.
KIE_DEV void prefetch_l1(const void *p) { asm volatile("prefetch.global.L1 [%0];" ::"l"(p)); }

// Hint: bring the 128-byte line holding p into L2 (through the load/store unit).
KIE_DEV void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// Hint: bring [src, src + bytes) into L2 (no completion tracking). bytes a multiple of 16.
KIE_DEV void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ------------------------------------------------------------------ storage types

// two stored elements packed in a 32-bit word -> two floats (low half first)
template <int DT>
KIE_DEV void cvt2(uint32_t w, float &lo, float &hi) {
    if (DT == KIE_BF16) {
        lo = __uint_as_float(w << 16);
        hi = __uint_as_float(w & 0xFFFF0000u);
    } else {
        lo = __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu)));
        hi = __half2float(__ushort_as_half((unsigned short)(w >> 16)));
    }
}

// 8 stored elements (one 16-byte vector) -> 8 floats.
template <int DT>
KIE_DEV void cvt8(const uint4 &v, float *f) {
    cvt2<DT>(v.x, f[0], f[1]);
    cvt2<DT>(v.y, f[2], f[3]);
    cvt2<DT>(v.z, f[4], f[5]);
    cvt2<DT>(v.w, f[6], f[7]);
}

template <int DT>
KIE_DEV float cvt1(uint16_t b) {
    if (DT == KIE_BF16) return __uint_as_float((uint32_t)b << 16);
    return __half2float(__ushort_as_half(b));
}

// float -> storage element, round to nearest even.
template <int DT>
KIE_DEV uint16_t store1(float f) {
    if (DT == KIE_BF16) return __bfloat16_as_ushort(__float2bfloat16_rn(f));
    return __half_as_ushort(__float2half_rn(f));
}

// byte offset of 16-byte chunk c (0..7) of row r in a 128 x 64 16-bit tile stored K-major with
// the 128-byte swizzle (8-row atoms of 1024 B; the MMA operand layout of the tick kernel)
KIE_DEV uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// make this thread's generic-proxy global writes visible to later async-proxy (bulk copy)
// reads, and order its async-proxy reads after its earlier generic accesses
KIE_DEV void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

KIE_DEV float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

KIE_DEV float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Reduces R partial sums (R in 1,2,4,8) across the warp. Afterwards lane l holds the full
// sum of row l / (32 / R) (every lane of that row group holds it).
template <int R>
KIE_DEV float warp_reduce_rows(float (&acc)[8]) {
    const int lane = threadIdx.x & 31;
    int n = R;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        if (n > 1) {
            const bool hi = (lane & off) != 0;
            const int h = n >> 1;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                if (j < h) {
                    float send = hi ? acc[j] : acc[j + h];
                    float keep = hi ? acc[j + h] : acc[j];
                    acc[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
            n = h;
        } else {
            acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], off);
        }
    }
    return acc[0];
}
