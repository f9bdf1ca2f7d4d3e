// k_cache_write.cu -- the cache-writing stage's copy into the ring and the spatial cache.
//
// Ca2-VDM ("Ca2-VDM" papernotes page, 整体框架 and 关键设计 4-5): after a chunk is denoised,
// one clean forward pass computes its K/V, which join the temporal queue (FIFO, at most
// Pmax frames) and replace the one-chunk spatial cache.  This kernel is the data movement
// of that step for every layer at once: a bit-exact copy, 16 bytes per access.  The ring
// is token-major and head-major within a token ([B][HW][H][Pmax][D]: one head's Pmax slots
// are contiguous), so a temporal write moves each (token, frame, head) row of D elements of
// the chunk into that head's slot.
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

// blockIdx.y = (layer, tensor): tensor 0/1 = temporal K/V, 2/3 = spatial K/V.
//   temporal: chunk [B][HW][n][H][D] -> ring [B][HW][H][Pmax][D]; (token, j, h) -> slot (slot0 + j) mod Pmax
//   spatial : chunk [B][n][HW][C], its last n_sp frames -> spatial cache [n_sp][B][HW][C]
//   (K copied, V converted to fp16)
// (source rows are src_row_vec 16-byte vectors apart, of which the first row_vec are copied)
__global__ void __launch_bounds__(kThreads) k_cache_write(const CacheWriteParams p)
{
    const int li = blockIdx.y >> 2;
    const int tensor = blockIdx.y & 3;
    const CacheWriteLayer &Ly = p.layer[li];
    const long long layer = p.layer0 + li;
    const long long rv = p.row_vec;
    long long total;
    const uint4 *src;
    uint4 *dst;
    if (tensor < 2) {
        total = p.tokens * p.n * rv;
        src = tensor == 0 ? Ly.kt : Ly.vt;
        dst = p.tbuf + ((layer * 2 + tensor) * p.tokens) * p.p_max * rv;
    } else {
        total = (long long)p.n_sp * p.tokens * rv;
        src = tensor == 2 ? Ly.ks : Ly.vs;
        dst = p.sbuf + ((layer * 2 + (tensor - 2)) * p.p_spatial) * p.tokens * rv;
    }
    const long long base = (long long)blockIdx.x * (kThreads * kVecPerThread) + threadIdx.x;
    if (base >= total) return;
    uint4 v[kVecPerThread];
    long long so[kVecPerThread], dof[kVecPerThread];
#pragma unroll
    for (int i = 0; i < kVecPerThread; ++i) {
        const long long e = base + (long long)i * kThreads;
        so[i] = dof[i] = -1;
        if (e < total) {
            const long long row = e / rv, off = e - row * rv;
            if (tensor < 2) {
                const long long tok = row / p.n;
                const int j = (int)(row - tok * p.n);
                int slot = p.slot0 + j;
                if (slot >= p.p_max) slot -= p.p_max;
                const int h = (int)(off / p.head_vec);
                const long long dv = off - (long long)h * p.head_vec;
                so[i] = row * p.src_row_vec + off;
                dof[i] = ((tok * p.heads + h) * p.p_max + slot) * p.head_vec + dv;
            } else {
                // row = jsp * tokens + (b * HW + s); source frame n - n_sp + jsp of video b
                const long long jsp = row / p.tokens;
                const long long bt = row - jsp * p.tokens;
                const long long b = bt / p.hw, sidx = bt - b * p.hw;
                so[i] = ((b * p.n + (p.n - p.n_sp + jsp)) * p.hw + sidx) * p.src_row_vec + off;
                dof[i] = e;
            }
            v[i] = ld_stream(src + so[i]);
        }
    }
    if (tensor & 1) {
        // both caches keep V in fp16, the operand type of the attention's P V products: the
        // exact value of each bf16 element within the fp16 range; elements beyond it
        // (|v| >= 65536, inf, NaN) are recorded as a range error
        uint32_t vmax = 0;
#pragma unroll
        for (int i = 0; i < kVecPerThread; ++i) {
            if (dof[i] < 0) continue;
            vmax = __vmaxu2(vmax, abs_max4(v[i].x, v[i].y, v[i].z, v[i].w));
            v[i] = make_uint4(pack_f16x2(bf16_lo(v[i].x), bf16_hi(v[i].x)), pack_f16x2(bf16_lo(v[i].y), bf16_hi(v[i].y)),
                              pack_f16x2(bf16_lo(v[i].z), bf16_hi(v[i].z)), pack_f16x2(bf16_lo(v[i].w), bf16_hi(v[i].w)));
        }
        if ((vmax & 0xFFFFu) >= 0x4780u || (vmax >> 16) >= 0x4780u) record_status(kStatusRange);
    }
#pragma unroll
    for (int i = 0; i < kVecPerThread; ++i)
        if (dof[i] >= 0) dst[dof[i]] = v[i];
}

cudaError_t launch_cache_write(const CacheWriteParams &p, cudaStream_t stream)
{
    const long long per_block = (long long)kThreads * kVecPerThread;
    const long long t_total = p.tokens * p.n * p.row_vec;
    const long long s_total = (long long)p.n_sp * p.tokens * p.row_vec;
    const long long most = t_total > s_total ? t_total : s_total;
    dim3 grid((unsigned)((most + per_block - 1) / per_block), (unsigned)(p.n_layers * 4));
    if (grid.x == 0 || grid.y == 0) return cudaSuccess;
    // a plain launch: it starts only after the previous kernel on the stream (the last
    // attention pass reads the cache) has completed
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
