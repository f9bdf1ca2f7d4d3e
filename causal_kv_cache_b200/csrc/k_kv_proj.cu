// k_kv_proj.cu -- the K/V projection of the cache-writing stage, with the cache write in its
// epilogue (sm_100a, tcgen05).
//
// Ca2-VDM ("Ca2-VDM" papernotes page, 整体框架: the cache-writing stage runs one forward
// pass over the denoised chunk and stores the new KV cache; 关键设计 4 and 5: the temporal
// queue and the one-chunk spatial cache).  For one layer:
//   temporal: row (b, s, f) of x_t [B][HW][n][C] -> [K | V] = x_t W_t^T + b_t, stored in
//             ring slot (slot0 + f) mod Pmax of token (b, s) -- the ring's own layout;
//   spatial : row s of frame f of x_s [B][n][HW][C], f among the chunk's last n_sp frames
//             -> [K | V] = x_s W_s^T + b_s, stored in spatial-cache frame f - (n - n_sp).
// The projections never exist as a tensor of their own: each 128-row x 192-channel output
// tile is accumulated in TMEM and written from registers straight to its cache rows, so
// the separate cache write (a read and a write of every K and V) disappears.
//
// One CTA per output tile; the temporal and spatial tiles share one grid.  Four warps:
//   warp 0   TMA producer: per 64-channel k-step an A tile (128 rows) and a W tile (192
//            output channels), 128-byte rows with the 128-byte swizzle, kStages deep.
//   warp 1   MMA issuer (whole warp, one elected lane): per k-step four tcgen05.mma of
//            M = 128, N = 192, K = 16 into a 192-column fp32 accumulator in TMEM.
//   all 4    epilogue: warp w reads TMEM lanes 32w..32w+31 (its 32 rows), 32 columns at
//            a time, adds the bias, rounds to bf16 (nearest, ties to even) and stores
//            16-byte pieces of 8 channels; a piece never crosses a head because D and C
//            are multiples of 8.
// Channels past C in a k-step, rows past the end and output channels past 2C are
// zero-filled by the TMA unit; the epilogue skips rows and channels that do not exist.
// Every mbarrier wait is bounded; a timeout is recorded in the library status word.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ca2_device.cuh"
#include "ca2_kernels.h"
#include "ca2_tcgen05.cuh"

namespace ca2 {

namespace {

constexpr int kThreads = 128;
constexpr int kBM = 128;                                  // rows per tile (TMEM lanes)
constexpr int kBN = kProjBN;                              // output channels per tile (TMEM columns)
constexpr int kBK = 64;                                   // input channels per k-step (128-byte rows)
constexpr int kStages = kProjStages;
constexpr uint32_t kATile = kBM * kBK * 2;                // 16 KB
constexpr uint32_t kWTile = kBN * kBK * 2;                // 24 KB
constexpr uint32_t kStageBytes = kATile + kWTile;
constexpr uint32_t kTmemCols = kBN <= 32 ? 32u : kBN <= 64 ? 64u : kBN <= 128 ? 128u : 256u;   // power of 2
constexpr uint32_t kSw128 = 2;                            // smem-descriptor layout code: 128-byte swizzle
constexpr uint32_t kBarBytes = 8u * (2 * kStages + 1) + 16u;   // barriers, abort flag, TMEM address
constexpr uint32_t kSmemBytes = kStages * kStageBytes + kBarBytes + 1024u;   // + base alignment

// the bias of 8 consecutive channels (16 bytes), or zeros
__device__ __forceinline__ void bias8(const __nv_bfloat16 *b, int ch, float (&f)[8])
{
    if (b) {
        const uint4 v = *reinterpret_cast<const uint4 *>(b + ch);
        f[0] = bf16_lo(v.x), f[1] = bf16_hi(v.x), f[2] = bf16_lo(v.y), f[3] = bf16_hi(v.y);
        f[4] = bf16_lo(v.z), f[5] = bf16_hi(v.z), f[6] = bf16_lo(v.w), f[7] = bf16_hi(v.w);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = 0.f;
    }
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) k_kv_proj(const __grid_constant__ KvProjMaps tm, const KvProjParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;           // 1024-aligned for the swizzled tiles
    uint8_t *sgen = smem_raw + (sb - raw);
    const uint32_t bars = sb + kStages * kStageBytes;
    auto full_bar = [&](int s) { return bars + 8u * (uint32_t)s; };
    auto empty_bar = [&](int s) { return bars + 8u * (uint32_t)(kStages + s); };
    const uint32_t acc_bar = bars + 8u * (uint32_t)(2 * kStages);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sgen + kStages * kStageBytes + 8 * (2 * kStages + 1));
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sgen + kStages * kStageBytes + 8 * (2 * kStages + 1) + 8);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // tile -> problem, row tile, channel tile (and for a spatial tile: video, frame)
    int t = blockIdx.x;
    const bool spatial = t >= p.tiles_t;
    if (spatial) t -= p.tiles_t;
    const int tn = t % p.tiles_n;
    t /= p.tiles_n;
    int tm_row = t, jsp = 0, vid = 0, plane = 0;
    if (spatial) {
        tm_row = t % p.tiles_s_frame;
        t /= p.tiles_s_frame;
        jsp = t % p.n_sp;                                 // spatial-cache frame
        vid = t / p.n_sp;
        plane = vid * p.n + (p.n - p.n_sp) + jsp;         // frame of x_s read
    }
    const CUtensorMap *ma = spatial ? &tm.xs : &tm.xt;
    const CUtensorMap *mw = spatial ? &tm.ws : &tm.wt;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(acc_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(ma);
        prefetch_tmap(mw);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32((const void *)tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // the previous kernel on the stream has completed: inputs may now be read
    wait_previous_kernel();
    allow_next_kernel();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------- TMA producer -------------------------------
        int issued = -1;
        for (int ks = 0; ks < p.k_steps; ++ks) {
            const int s = ks % kStages;
            if (ks >= kStages && !warp_wait(empty_bar(s), ((ks / kStages) - 1) & 1, 301, abort_flag)) break;
            if (lane == 0) {
                const uint32_t a = sb + (uint32_t)s * kStageBytes;
                mbar_expect_tx(full_bar(s), kStageBytes);
                tma_load_3d(a, ma, ks * kBK, tm_row * kBM, plane, full_bar(s));
                tma_load_3d(a + kATile, mw, ks * kBK, tn * kBN, 0, full_bar(s));
            }
            issued = ks;
            __syncwarp();
        }
        // wind-down after an abort: the issued loads land before the CTA exits
        if (lane == 0 && *abort_flag)
            for (int ks = issued; ks >= 0 && ks > issued - kStages; --ks)
                mbar_wait(full_bar(ks % kStages), (ks / kStages) & 1, 0, nullptr, 2000000ull);
    } else if (warp == 1) {
        // ------------------------------- MMA issuer ---------------------------------
        // K-major operands with the 128-byte swizzle: 8-row groups 1024 B apart; the k-step
        // kk of 16 channels starts 32 B further into each 128-byte row.
        constexpr uint32_t idesc = idesc_bf16(kBM, kBN, false, false);
        const uint32_t tm_u = __shfl_sync(0xffffffffu, tmem, 0);
        for (int ks = 0; ks < p.k_steps; ++ks) {
            const int s = ks % kStages;
            if (!warp_wait(full_bar(s), (ks / kStages) & 1, 302, abort_flag)) break;
            tc_fence_after();
            const uint32_t a = sb + (uint32_t)s * kStageBytes;
            const uint64_t da = sdesc(a, 16, 1024, kSw128);
            const uint64_t dw = sdesc(a + kATile, 16, 1024, kSw128);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
                tc_mma_ss_w(tm_u, da + (uint64_t)(2 * kk), dw + (uint64_t)(2 * kk), idesc, (ks > 0 || kk > 0) ? 1u : 0u);
            tc_commit_w(empty_bar(s));
        }
        // fires once every issued MMA has completed (after an abort too); this warp frees
        // TMEM, so it waits for that itself, bounded and regardless of the abort flag
        tc_commit_w(acc_bar);
        mbar_wait(acc_bar, 0, 0, nullptr, 2000000ull);
        __syncwarp();
    }

    // ------------------------------- epilogue (all warps) ---------------------------------
    __syncwarp();
    const bool acc_ok = warp_wait(acc_bar, 0, 303, abort_flag);
    if (acc_ok && !*abort_flag) {
        tc_fence_after();
        const int r = warp * 32 + lane;                   // row of the tile = TMEM lane
        // row -> element offset of the row's (h = 0, d = 0) in its cache, and the stride
        // between consecutive heads
        long long base = -1;
        long long head_stride = 0;
        if (!spatial) {
            const int m = tm_row * kBM + r;
            if (m < p.rows_t) {
                const int f = m % p.n;
                const long long bs = m / p.n;             // b * HW + s
                const int slot = (p.slot0 + f) % p.p_max;
                base = (bs * p.H * p.p_max + slot) * (long long)p.D;
                head_stride = (long long)p.p_max * p.D;
            }
        } else {
            const int s = tm_row * kBM + r;
            if (s < p.HW) {
                base = (((long long)jsp * p.B + vid) * p.HW + s) * (long long)p.H * p.D;
                head_stride = p.D;
            }
        }
        const __nv_bfloat16 *bias = spatial ? p.bias_s : p.bias_t;
        __nv_bfloat16 *dst_k = spatial ? p.sp_k : p.ring_k;
        __nv_bfloat16 *dst_v = spatial ? p.sp_v : p.ring_v;
        const uint32_t lane_bits = (uint32_t)(warp * 32) << 16;
        for (int c0 = 0; c0 < kBN; c0 += 32) {
            const int n0 = tn * kBN + c0;
            if (n0 >= 2 * p.C) break;                     // warp-uniform
            uint32_t v[32];
            tmem_ld32(tmem + lane_bits + (uint32_t)c0, v);
            if (base < 0) continue;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int ch = n0 + 8 * q;
                if (ch >= 2 * p.C) break;
                const int kv = ch >= p.C ? 1 : 0;
                const int rem = ch - kv * p.C;
                const int h = rem / p.D;
                const int d = rem - h * p.D;
                float b8[8];
                bias8(bias, ch, b8);
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) + b8[0], __uint_as_float(v[8 * q + 1]) + b8[1]);
                w.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) + b8[2], __uint_as_float(v[8 * q + 3]) + b8[3]);
                w.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) + b8[4], __uint_as_float(v[8 * q + 5]) + b8[5]);
                w.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) + b8[6], __uint_as_float(v[8 * q + 7]) + b8[7]);
                __nv_bfloat16 *dst = (kv ? dst_v : dst_k) + base + (long long)h * head_stride + d;
                *reinterpret_cast<uint4 *>(dst) = w;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

cudaError_t launch_kv_proj(const KvProjMaps &m, const KvProjParams &p, int grid, cudaStream_t stream)
{
    static int configured_for = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_for != dev) {
        cudaError_t e = cudaFuncSetAttribute(k_kv_proj, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        configured_for = dev;
    }
    if (grid <= 0) return cudaSuccess;
    return launch_chained(k_kv_proj, dim3((unsigned)grid), dim3(kThreads), kSmemBytes, stream, m, p);
}

}  // namespace ca2
