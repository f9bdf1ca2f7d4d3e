// k_cache_write.cu -- the cache-writing stage's copy into the ring and the spatial cache.
//
// Ca2-VDM ("Ca2-VDM" papernotes page, 整体框架 and 关键设计 4-5): after a chunk is denoised,
// one clean forward pass computes its K/V, which join the temporal queue (FIFO, at most
// Pmax frames) and replace the one-chunk spatial cache.  This kernel is the data movement
// of that step for every layer at once: a bit-exact copy of frame-planes, 16 bytes per
// access, one block row per (layer, tensor, video, frame) copy.
#include <cstdint>

#include "ca2_device.cuh"
#include "ca2_kernels.h"

namespace ca2 {

__device__ int g_status = 0;

namespace {
constexpr int kThreads = 256;
constexpr int kVecPerThread = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
}  // namespace

__global__ void __launch_bounds__(kThreads) k_cache_write(const CacheWriteParams p)
{
    // blockIdx.y enumerates copies: per layer, B * (2n + 2 n_sp) of them
    const int per_layer = p.B * (2 * p.n + 2 * p.n_sp);
    const int cy = blockIdx.y;
    const int li = cy / per_layer;
    const int r = cy - li * per_layer;
    const int t = r / p.B;          // which frame of which tensor
    const int b = r - t * p.B;
    const CacheWriteLayer &Ly = p.layer[li];
    const int layer = p.layer0 + li;

    const uint4 *src;
    uint4 *dst;
    if (t < 2 * p.n) {
        const int kv = t >= p.n;
        const int j = kv ? t - p.n : t;
        int slot = p.slot0 + j;
        if (slot >= p.p_max) slot -= p.p_max;
        src = (kv ? Ly.vt : Ly.kt) + ((long long)b * p.n + j) * p.plane_vec;
        dst = p.tbuf + ((((long long)layer * 2 + kv) * p.p_max + slot) * p.B + b) * p.plane_vec;
    } else {
        const int u = t - 2 * p.n;
        const int kv = u >= p.n_sp;
        const int jsp = kv ? u - p.n_sp : u;             // spatial slot, oldest first
        const int j = p.n - p.n_sp + jsp;                // frame of the chunk
        src = (kv ? Ly.vs : Ly.ks) + ((long long)b * p.n + j) * p.plane_vec;
        dst = p.sbuf + ((((long long)layer * 2 + kv) * p.p_spatial + jsp) * p.B + b) * p.plane_vec;
    }

    const long long base = (long long)blockIdx.x * (kThreads * kVecPerThread) + threadIdx.x;
    uint4 v[kVecPerThread];
#pragma unroll
    for (int i = 0; i < kVecPerThread; ++i) {
        const long long e = base + (long long)i * kThreads;
        if (e < p.plane_vec) v[i] = ld_stream(src + e);
    }
#pragma unroll
    for (int i = 0; i < kVecPerThread; ++i) {
        const long long e = base + (long long)i * kThreads;
        if (e < p.plane_vec) dst[e] = v[i];
    }
}

cudaError_t launch_cache_write(const CacheWriteParams &p, cudaStream_t stream)
{
    const long long per_block = (long long)kThreads * kVecPerThread;
    dim3 grid((unsigned)((p.plane_vec + per_block - 1) / per_block),
              (unsigned)(p.n_layers * p.B * (2 * p.n + 2 * p.n_sp)));
    if (grid.x == 0 || grid.y == 0) return cudaSuccess;
    k_cache_write<<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

// ---- bounded-wait self test -------------------------------------------------------------
// One block waits on an mbarrier that nothing will ever complete, gives up after limit_ns,
// records the timeout in the status word and returns normally.
__global__ void k_timeout_selftest(unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, 999, &abort_flag, limit_ns);
    __syncthreads();
}

cudaError_t launch_timeout_selftest(unsigned long long limit_ns, cudaStream_t stream)
{
    k_timeout_selftest<<<1, 32, 0, stream>>>(limit_ns);
    return cudaGetLastError();
}

int read_and_clear_status(int *status)
{
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(status, g_status, sizeof(int));
    if (e != cudaSuccess) return (int)e;
    e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
    return (int)e;
}

}  // namespace ca2
