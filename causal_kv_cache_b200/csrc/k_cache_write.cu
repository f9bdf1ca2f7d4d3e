// k_cache_write.cu -- the cache-writing stage's copy into the ring and the spatial cache.
//
// Ca2-VDM ("Ca2-VDM" papernotes page, 整体框架 and 关键设计 4-5): after a chunk is denoised,
// one clean forward pass computes its K/V, which join the temporal queue (FIFO, at most
// Pmax frames) and replace the one-chunk spatial cache.  This kernel is the data movement
// of that step for every layer at once: a copy, 16 bytes per access (K bit for bit, V as
// the exact fp16 form of each bf16 value).  The ring is token-major and head-major within a
// token ([B][HW][H][Pmax][D]: one head's Pmax slots are contiguous), so a temporal write
// moves the chunk's n rows of D elements of each (token, head) into n consecutive slots of
// that head.
#include <cstdint>

#include "ca2_device.cuh"
#include "ca2_kernels.h"

namespace ca2 {

__device__ int g_status = 0;

namespace {
constexpr int kThreads = 256;
constexpr int kUnroll = 4;        // loads in flight per lane

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
// The copy is cut into runs that are contiguous in the destination:
//   temporal: run (token, h) = head h of the chunk's n rows of that token -> the head's n
//             consecutive ring slots (slot0 + j) mod Pmax: n * head_vec vectors (two pieces
//             when the slots wrap past Pmax);
//   spatial : run (jsp, b, s) = one row of the chunk's frame n - n_sp + jsp -> one row of the
//             spatial cache [n_sp][B][HW][C].
// A warp takes whole runs (grid-stride over the runs) and its lanes take a run's vectors in
// order, 32 at a time, so a warp's stores cover up to 512 contiguous bytes: the ring's
// 32-byte sectors are written whole except at a run's two ends.  Each lane keeps up to
// kUnroll loads in flight.  K is copied; V is converted to fp16.  Source rows are
// src_row_vec 16-byte vectors apart.
__global__ void __launch_bounds__(kThreads) k_cache_write(const CacheWriteParams p)
{
    const int li = blockIdx.y >> 2;
    const int tensor = blockIdx.y & 3;
    const CacheWriteLayer &Ly = p.layer[li];
    const long long layer = p.layer0 + li;
    const int lane = threadIdx.x & 31;
    const long long warp0 = ((long long)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const long long n_warps = (long long)gridDim.x * (kThreads / 32);
    const bool is_v = (tensor & 1) != 0;
    uint32_t vmax = 0;       // max |v| bits per half, V tensors only

    // V: the fp16 form of each bf16 element (exact within the fp16 range); elements beyond it
    // (|v| >= 65536, inf, NaN) are recorded as a range error below
    auto to_f16 = [&](uint4 &x) {
        vmax = __vmaxu2(vmax, abs_max4(x.x, x.y, x.z, x.w));
        x = make_uint4(pack_f16x2(bf16_lo(x.x), bf16_hi(x.x)), pack_f16x2(bf16_lo(x.y), bf16_hi(x.y)),
                       pack_f16x2(bf16_lo(x.z), bf16_hi(x.z)), pack_f16x2(bf16_lo(x.w), bf16_hi(x.w)));
    };

    if (tensor < 2) {
        const uint4 *src = tensor == 0 ? Ly.kt : Ly.vt;
        const long long dst0 = ((layer * 2 + tensor) * p.tokens) * p.p_max * p.row_vec;
        uint4 *dst = p.tbuf + dst0;
        const int hv = p.head_vec;
        const int run_len = p.n * hv;
        const long long runs = p.tokens * p.heads;
        // (frame, vector) of a run position: this lane's first, and the step of 32 positions
        const int j_first = lane / hv, dv_first = lane - (lane / hv) * hv;
        const int dj = 32 / hv, ddv = 32 - (32 / hv) * hv;
        for (long long r = warp0; r < runs; r += n_warps) {
            const long long tok = r / p.heads;
            const int h = (int)(r - tok * p.heads);
            const long long s0 = tok * p.n * p.src_row_vec + (long long)h * hv;
            const long long d0 = r * p.p_max * hv;
            const uint4 *s = src + s0;
            uint4 *d = dst + d0;
            int j = j_first, dv = dv_first;
            for (int q = lane; q < run_len; q += 32 * kUnroll) {
                uint4 v[kUnroll];
                int doff[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    doff[u] = -1;
                    if (q + 32 * u < run_len) {
                        const long long so = (long long)j * p.src_row_vec + dv;
                        v[u] = CA2_IN_BOUNDS(s0 + so < p.t_src_vec, 21) ? ld_stream(s + so) : make_uint4(0u, 0u, 0u, 0u);
                        int slot = p.slot0 + j;
                        if (slot >= p.p_max) slot -= p.p_max;
                        doff[u] = slot * hv + dv;
                        if (!CA2_IN_BOUNDS(dst0 + d0 + doff[u] < p.tbuf_vec, 22)) doff[u] = -1;
                    }
                    dv += ddv;
                    j += dj;
                    if (dv >= hv) { dv -= hv; ++j; }
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    if (doff[u] < 0) continue;
                    if (is_v) to_f16(v[u]);
                    d[doff[u]] = v[u];
                }
            }
        }
    } else {
        const uint4 *src = tensor == 2 ? Ly.ks : Ly.vs;
        const long long dst0 = ((layer * 2 + (tensor - 2)) * p.p_spatial) * p.tokens * p.row_vec;
        uint4 *dst = p.sbuf + dst0;
        const int rv = (int)p.row_vec;
        const long long runs = (long long)p.n_sp * p.tokens;
        for (long long r = warp0; r < runs; r += n_warps) {
            // r = jsp * tokens + (b * HW + s): source frame n - n_sp + jsp of video b
            const long long jsp = r / p.tokens;
            const long long bt = r - jsp * p.tokens;
            const long long b = bt / p.hw, sidx = bt - b * p.hw;
            const long long s0 = ((b * p.n + (p.n - p.n_sp + jsp)) * p.hw + sidx) * p.src_row_vec;
            const uint4 *s = src + s0;
            uint4 *d = dst + r * rv;
            for (int q = lane; q < rv; q += 32 * kUnroll) {
                uint4 v[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u)
                    if (q + 32 * u < rv)
                        v[u] = CA2_IN_BOUNDS(s0 + q + 32 * u < p.s_src_vec, 23) ? ld_stream(s + q + 32 * u)
                                                                               : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    if (q + 32 * u >= rv) continue;
                    if (!CA2_IN_BOUNDS(dst0 + r * rv + q + 32 * u < p.sbuf_vec, 24)) continue;
                    if (is_v) to_f16(v[u]);
                    d[q + 32 * u] = v[u];
                }
            }
        }
    }
    if (is_v && ((vmax & 0xFFFFu) >= 0x4780u || (vmax >> 16) >= 0x4780u)) record_status(kStatusRange);
}

cudaError_t launch_cache_write(const CacheWriteParams &p, cudaStream_t stream)
{
    // about two temporal runs per warp; the spatial blocks of the same grid stride over fewer
    const long long t_runs = p.tokens * p.heads;
    const long long s_runs = (long long)p.n_sp * p.tokens;
    const long long warps = (t_runs + 1) / 2 > s_runs ? (t_runs + 1) / 2 : s_runs;
    const long long gx = (warps + kThreads / 32 - 1) / (kThreads / 32);
    dim3 grid((unsigned)(gx < 65535 ? gx : 65535), (unsigned)(p.n_layers * 4));
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
