// ca2_device.cuh -- device-side building blocks shared by the libca2 kernels (sm_100a).
//
// mbarrier waits here are bounded: a wait that runs past its limit records a code in the
// library's device status word (read by ca2_device_status) and returns false, so a kernel
// can wind down instead of spinning forever.  Nothing here traps.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace ca2 {

// Device status word: 0 = fine, otherwise the site code of the first wait that gave up.
extern __device__ int g_status;

// Wait limit in nanoseconds of %globaltimer (about one second).
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void record_timeout(int site)
{
    atomicCAS(&g_status, 0, site);
}

// Status codes of kStatusRange and above mean an input outside the supported range (not a
// timeout); the first record wins, as for timeouts.  (The same value as kStatusRangeCode,
// which the host side reads.)
constexpr int kStatusRange = 1000;
__device__ __forceinline__ void record_status(int code)
{
    atomicCAS(&g_status, 0, code);
}

// Bounds checks of the debug build (compiled with -DCA2_DEBUG, libca2_debug.so): every
// global access a kernel addresses itself (plain loads and stores, bulk copies) is checked
// against the extent of its buffer.  A failed check records kStatusBounds + site and the
// access is skipped; nothing traps.  Release builds compile the checks out (the condition is
// not evaluated).  Accesses through tensor maps are bounded by the maps' extents, which the
// TMA unit enforces in both builds.  (The same value as kStatusBoundsCode on the host side.)
constexpr int kStatusBounds = 2000;
#ifdef CA2_DEBUG
#define CA2_IN_BOUNDS(cond, site) \
    ((cond) ? true : (::ca2::record_status(::ca2::kStatusBounds + (site)), false))
#else
#define CA2_IN_BOUNDS(cond, site) true
#endif

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier -----------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete.  Gives up after limit_ns (or at
// once when *abort is set by another warp of the CTA), records `site`, returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int site,
                                          volatile int *abort,
                                          unsigned long long limit_ns = kWaitLimitNs)
{
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (abort && *abort) return false;
            if (global_ns() - t0 > limit_ns) {
                record_timeout(site);
                if (abort) *abort = 1;
                return false;
            }
        }
    }
}

// Warp-wide wait: every lane polls (so every lane acquires the phase), and the outcome
// is made uniform so that a warp never splits on a timeout.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int site, volatile int *abort)
{
    const bool ok = mbar_wait(bar, parity, site, abort);
    return __all_sync(0xffffffffu, ok);
}

// ---- programmatic dependent launch ------------------------------------------------------
// The attention kernels are launched so that the next kernel on the stream may start while
// this one drains.  Each kernel does its set-up (barriers, TMEM, tensor-map prefetch), then
// every thread waits for the previous kernel on the stream to complete (its memory visible)
// before touching global memory, and only then lets its own dependent start: so a kernel's
// set-up never overlaps anything but its immediate predecessor's last CTAs.
__device__ __forceinline__ void wait_previous_kernel() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_next_kernel() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- work stealing between CTAs of one grid (cluster launch control) ---------------
// Ask the hardware to cancel the launch of a CTA of this grid that has not started yet; the
// 16-byte response lands in shared memory and completes 16 bytes of transaction on `bar`.
// After a response that reports failure, no further request may be made.
__device__ __forceinline__ void work_request(uint32_t resp, uint32_t bar)
{
    asm volatile("clusterlaunchcontrol.try_cancel.async.shared::cta.mbarrier::complete_tx::bytes.b128 [%0], [%1];"
                 ::"r"(resp), "r"(bar)
                 : "memory");
}
// Decode a response: true and the cancelled CTA's x index, or false (no CTA left to take).
__device__ __forceinline__ bool work_response(uint32_t resp, uint32_t &ctaid_x)
{
    uint32_t ok, x;
    asm volatile("{\n\t.reg .pred p;\n\t.reg .b128 r;\n\t"
                 "ld.shared.b128 r, [%2];\n\t"
                 "clusterlaunchcontrol.query_cancel.is_canceled.pred.b128 p, r;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t"
                 "clusterlaunchcontrol.query_cancel.get_first_ctaid::x.b32.b128 %1, r;\n\t}"
                 : "=r"(ok), "=r"(x)
                 : "r"(resp)
                 : "memory");
    ctaid_x = x;
    return ok != 0;
}

// ---- bulk copies (TMA engine) --------------------------------------------------------
// 1-D bulk copy global -> shared, completing `bytes` of transaction on an mbarrier.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Hint: bring `bytes` of global memory into L2 (16-byte aligned address and size).  A
// prefetch only moves data into L2, the point of coherence, so it may run before the
// previous kernel's writes are complete: later loads still see the current values.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// 1-D bulk copy shared -> global (bulk-group completion).
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait()
{
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Tiled 4-D tensor load (no multicast), completing on an mbarrier.
// Tiled 3-D tensor load into shared memory, completing on an mbarrier.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void *tmap, int c0, int c1, int c2, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void *tmap, int c0, int c1, int c2, int c3,
                                            uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
        "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
        : "memory");
}

// Tiled 4-D tensor store (bulk-group completion).  Out-of-range rows are not written.
__device__ __forceinline__ void tma_store_4d(const void *tmap, uint32_t src, int c0, int c1, int c2, int c3)
{
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                     tmap),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void *tmap)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async proxy
// (bulk copies, tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// The two bf16 halves of a packed word, widened exactly to fp32.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Per-halfword maximum of the magnitude bits of four words of bf16 pairs (the sign bit is
// cleared before the max, so a negative value never hides a larger magnitude).
__device__ __forceinline__ uint32_t abs_max4(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return __vmaxu2(__vmaxu2(a & 0x7FFF7FFFu, b & 0x7FFF7FFFu), __vmaxu2(c & 0x7FFF7FFFu, d & 0x7FFF7FFFu));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    __half2 v = __floats2half2_rn(lo, hi);              // .x = lo (low half), .y = hi
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x = lo (low half), .y = hi
    return *reinterpret_cast<uint32_t *>(&v);
}

}  // namespace ca2
