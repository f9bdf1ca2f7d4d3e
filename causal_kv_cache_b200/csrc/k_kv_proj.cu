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
// Persistent: one CTA per SM walks the output tiles (temporal tiles first, then spatial)
// with a stride of the grid.  Six warps:
//   warp 0     TMA producer: per 64-channel k-step an A tile (128 rows) and a W tile (192
//              output channels), 128-byte rows with the 128-byte swizzle, into a ring of
//              kStages slots that runs on across tiles.
//   warp 1     MMA issuer (whole warp, one elected lane): per k-step four tcgen05.mma of
//              M = 128, N = 192, K = 16, into one of two fp32 TMEM accumulators (columns
//              0 and 256), alternating by tile.
//   warps 2-5  epilogue of the other accumulator while the next tile accumulates: warp w
//              reads TMEM lanes 32 (w % 4).. (its rows), 32 columns at a time, adds the
//              bias, rounds to bf16 (nearest, ties to even) and stores 16-byte pieces of 8
//              channels; a piece never crosses a head because D and C are multiples of 8.
// Channels past C in a k-step, rows past the end and output channels past 2C are
// zero-filled by the TMA unit; the epilogue skips rows and channels that do not exist.
// Every mbarrier wait is bounded; a timeout is recorded in the library status word and all
// roles wind down (issued copies land, issued MMAs complete, TMEM is freed).
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ca2_device.cuh"
#include "ca2_kernels.h"
#include "ca2_tcgen05.cuh"

namespace ca2 {

namespace {

constexpr int kThreads = 192;
constexpr int kBM = 128;                                  // rows per tile (TMEM lanes)
constexpr int kBN = kProjBN;                              // output channels per tile
constexpr int kBK = 64;                                   // input channels per k-step (128-byte rows)
constexpr int kStages = kProjStages;
constexpr uint32_t kAccStride = 256;                      // TMEM columns between the two accumulators
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kATile = kBM * kBK * 2;                // 16 KB
constexpr uint32_t kWTile = kBN * kBK * 2;                // 24 KB
constexpr uint32_t kStageBytes = kATile + kWTile;
constexpr uint32_t kSw128 = 2;                            // smem-descriptor layout code: 128-byte swizzle
// barriers: full[S], empty[S], acc_full[2], acc_empty[2], fin; then the abort flag and the
// TMEM address
constexpr int kBars = 2 * kStages + 5;
constexpr uint32_t kBarBytes = 8u * kBars + 16u;
constexpr uint32_t kSmemBytes = kStages * kStageBytes + kBarBytes + 1024u;   // + base alignment
static_assert(kBN <= (int)kAccStride && kAccStride + kBN <= kTmemCols, "accumulators overflow TMEM");
static_assert(kSmemBytes <= 232448u, "shared memory overflows");

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

// one output tile: problem, row tile, channel tile, and for a spatial tile the video and
// the spatial-cache frame (plane = frame of x_s read)
struct Tile {
    bool spatial;
    int tn, tm, jsp, vid, plane;
};

__device__ __forceinline__ Tile decode_tile(const KvProjParams &p, int t)
{
    Tile d{};
    d.spatial = t >= p.tiles_t;
    if (d.spatial) t -= p.tiles_t;
    d.tn = t % p.tiles_n;
    t /= p.tiles_n;
    d.tm = t;
    if (d.spatial) {
        d.tm = t % p.tiles_s_frame;
        t /= p.tiles_s_frame;
        d.jsp = t % p.n_sp;
        d.vid = t / p.n_sp;
        d.plane = d.vid * p.n + (p.n - p.n_sp) + d.jsp;
    }
    return d;
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
    auto acc_full = [&](int a) { return bars + 8u * (uint32_t)(2 * kStages + a); };
    auto acc_empty = [&](int a) { return bars + 8u * (uint32_t)(2 * kStages + 2 + a); };
    const uint32_t fin_bar = bars + 8u * (uint32_t)(2 * kStages + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sgen + kStages * kStageBytes + 8 * kBars);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sgen + kStages * kStageBytes + 8 * kBars + 8);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(acc_full(a), 1);
            mbar_init(acc_empty(a), 4);                   // the four epilogue warps
        }
        mbar_init(fin_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm.xt);
        prefetch_tmap(&tm.wt);
        prefetch_tmap(&tm.xs);
        prefetch_tmap(&tm.ws);
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
        int g = 0;                                        // k-steps issued by this CTA
        for (int t = blockIdx.x; t < p.total_tiles && !*abort_flag; t += gridDim.x) {
            const Tile d = decode_tile(p, t);
            const CUtensorMap *ma = d.spatial ? &tm.xs : &tm.xt;
            const CUtensorMap *mw = d.spatial ? &tm.ws : &tm.wt;
            bool ok = true;
            for (int ks = 0; ks < p.k_steps; ++ks, ++g) {
                const int s = g % kStages;
                if (g >= kStages && !warp_wait(empty_bar(s), ((g / kStages) - 1) & 1, 301, abort_flag)) { ok = false; break; }
                if (lane == 0) {
                    const uint32_t a = sb + (uint32_t)s * kStageBytes;
                    mbar_expect_tx(full_bar(s), kStageBytes);
                    tma_load_3d(a, ma, ks * kBK, d.tm * kBM, d.plane, full_bar(s));
                    tma_load_3d(a + kATile, mw, ks * kBK, d.tn * kBN, 0, full_bar(s));
                }
                __syncwarp();
            }
            if (!ok) break;
        }
        // wind-down after an abort: the issued loads land before the CTA exits
        if (lane == 0 && *abort_flag)
            for (int k = g - 1; k >= 0 && k >= g - kStages; --k)
                mbar_wait(full_bar(k % kStages), (k / kStages) & 1, 0, nullptr, 2000000ull);
    } else if (warp == 1) {
        // ------------------------------- MMA issuer ---------------------------------
        // K-major operands with the 128-byte swizzle: 8-row groups 1024 B apart; the k-step
        // kk of 16 channels starts 32 B further into each 128-byte row.
        constexpr uint32_t idesc = idesc_bf16(kBM, kBN, false, false);
        const uint32_t tm_u = __shfl_sync(0xffffffffu, tmem, 0);
        int g = 0, i = 0;                                 // k-steps and tiles of this CTA
        bool ok = true;
        for (int t = blockIdx.x; ok && t < p.total_tiles; t += gridDim.x, ++i) {
            const int acc = i & 1;
            // the epilogue of the tile that last used this accumulator is done with it
            if (i >= 2 && !warp_wait(acc_empty(acc), ((i >> 1) - 1) & 1, 304, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d_tmem = tm_u + (uint32_t)acc * kAccStride;
            for (int ks = 0; ks < p.k_steps; ++ks, ++g) {
                const int s = g % kStages;
                if (!warp_wait(full_bar(s), (g / kStages) & 1, 302, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a = sb + (uint32_t)s * kStageBytes;
                const uint64_t da = sdesc(a, 16, 1024, kSw128);
                const uint64_t dw = sdesc(a + kATile, 16, 1024, kSw128);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)
                    tc_mma_ss_w(d_tmem, da + (uint64_t)(2 * kk), dw + (uint64_t)(2 * kk), idesc,
                                (ks > 0 || kk > 0) ? 1u : 0u);
                tc_commit_w(empty_bar(s));
            }
            if (ok) tc_commit_w(acc_full(acc));
        }
        // every issued MMA completes before TMEM is freed (bounded, regardless of the abort)
        tc_commit_w(fin_bar);
        mbar_wait(fin_bar, 0, 0, nullptr, 2000000ull);
        __syncwarp();
    } else {
        // ------------------------------- epilogue (warps 2-5) --------------------------
        const int quarter = warp & 3;                     // TMEM lanes 32 * quarter ..
        const int r = quarter * 32 + lane;                // row of the tile = TMEM lane
        const uint32_t lane_bits = (uint32_t)(quarter * 32) << 16;
        uint32_t vmax = 0;                                // per-half max of the spatial V bits stored
        int i = 0;
        for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++i) {
            const int acc = i & 1;
            if (!warp_wait(acc_full(acc), (i >> 1) & 1, 303, abort_flag)) break;
            tc_fence_after();
            const Tile d = decode_tile(p, t);
            // row -> element offset of the row's (h = 0, d = 0) in its cache, and the stride
            // between consecutive heads
            long long base = -1;
            long long head_stride = 0;
            if (!d.spatial) {
                const int m = d.tm * kBM + r;
                if (m < p.rows_t) {
                    const int f = m % p.n;
                    const long long bs = m / p.n;         // b * HW + s
                    const int slot = (p.slot0 + f) % p.p_max;
                    base = (bs * p.H * p.p_max + slot) * (long long)p.D;
                    head_stride = (long long)p.p_max * p.D;
                }
            } else {
                const int s = d.tm * kBM + r;
                if (s < p.HW) {
                    base = (((long long)d.jsp * p.B + d.vid) * p.HW + s) * (long long)p.H * p.D;
                    head_stride = p.D;
                }
            }
            const __nv_bfloat16 *bias = d.spatial ? p.bias_s : p.bias_t;
            __nv_bfloat16 *dst_k = d.spatial ? p.sp_k : p.ring_k;
            __nv_bfloat16 *dst_v = d.spatial ? p.sp_v : p.ring_v;
            const uint32_t acc_cols = tmem + lane_bits + (uint32_t)acc * kAccStride;
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                const int n0 = d.tn * kBN + c0;
                if (n0 >= 2 * p.C) break;                 // warp-uniform
                uint32_t v[32];
                tmem_ld32(acc_cols + (uint32_t)c0, v);
                if (base < 0) continue;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int ch = n0 + 8 * q;
                    if (ch >= 2 * p.C) break;
                    const int kv = ch >= p.C ? 1 : 0;
                    const int rem = ch - kv * p.C;
                    const int h = rem / p.D;
                    const int dd = rem - h * p.D;
                    float b8[8];
                    bias8(CA2_IN_BOUNDS(ch + 8 <= 2 * p.C, 42) ? bias : nullptr, ch, b8);
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) + b8[0], __uint_as_float(v[8 * q + 1]) + b8[1]);
                    w.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) + b8[2], __uint_as_float(v[8 * q + 3]) + b8[3]);
                    w.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) + b8[4], __uint_as_float(v[8 * q + 5]) + b8[5]);
                    w.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) + b8[6], __uint_as_float(v[8 * q + 7]) + b8[7]);
                    if (kv) {
                        // both caches keep V in fp16: the exact value of the bf16 result within
                        // the fp16 range, larger values recorded as a range error
                        vmax = __vmaxu2(vmax, abs_max4(w.x, w.y, w.z, w.w));
                        w = make_uint4(pack_f16x2(bf16_lo(w.x), bf16_hi(w.x)), pack_f16x2(bf16_lo(w.y), bf16_hi(w.y)),
                                       pack_f16x2(bf16_lo(w.z), bf16_hi(w.z)), pack_f16x2(bf16_lo(w.w), bf16_hi(w.w)));
                    }
                    const long long off = base + (long long)h * head_stride + dd;
                    if (CA2_IN_BOUNDS(off + 8 <= (d.spatial ? p.sp_elems : p.ring_elems), 41))
                        *reinterpret_cast<uint4 *>((kv ? dst_v : dst_k) + off) = w;
                }
            }
            // the accumulator may take the tile after next
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty(acc));
        }
        if ((vmax & 0xFFFFu) >= 0x4780u || (vmax >> 16) >= 0x4780u) record_status(kStatusRange);
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
    static std::atomic<uint64_t> configured{0};
    const cudaError_t e = ensure_smem_attr(configured, reinterpret_cast<const void *>(&k_kv_proj), (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    if (grid <= 0) return cudaSuccess;
    return launch_chained(k_kv_proj, dim3((unsigned)grid), dim3(kThreads), kSmemBytes, stream, m, p);
}

}  // namespace ca2
