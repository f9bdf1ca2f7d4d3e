// ca2_kernels.h -- launch interface between the C-ABI layer (ca2_api.cu) and the kernels.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <utility>

namespace ca2 {

// Launch with programmatic stream serialization: the kernel may be scheduled while the
// previous kernel on the stream drains; it waits for that kernel (griddepcontrol.wait in
// every thread) before touching global memory.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                  Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raise a kernel's dynamic shared-memory limit on the current device, once per device.
// `configured` is the launch site's own record (bit d = done on device d); concurrent callers
// may both set the attribute, which is harmless.  Devices past 63 set it on every call.
inline cudaError_t ensure_smem_attr(std::atomic<uint64_t> &configured, const void *func, int bytes)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev >= 0 && dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (configured.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) configured.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// ---- causal temporal attention ---------------------------------------------------------
// heads per work item = consumer warps per CTA.  Two heads and four stages make CTAs of
// ~42 KB of shared memory at D = 72, five per SM: more independent consumer warps per SM
// measured faster than deeper rings in fewer CTAs (each consumer handles its stages one
// after another, so the number of consumers in flight sets the rate).
constexpr int kMaxTemporalGroup = 2;
constexpr int kMaxChunk = 8;           // queries per (token, head): the chunk length limit

struct TemporalParams {
    __nv_bfloat16 *out;                 // [B][HW][n][H][D]
    const uint8_t *rk, *rv;             // this layer's K and V rings [B][HW][H][Pmax][D]
    int B, HW, H, D;
    long long pitch;  // elements from one row of a chunk tensor to the next (>= H * D)
    int n;          // chunk frames in this call (queries per token-head)
    int Pk;         // queued frames
    int head;       // ring slot of the oldest queued frame
    int Pmax;
    int G;          // heads per work item
    int n_items;    // B * HW * (H / G)
    uint32_t ring_box_mask;   // bit i: ring slots [16i, 16i+16) hold at least one queued frame
    float scale_log2;         // log2(e) / sqrt(D)
    long long ring_bytes;     // bytes of one layer's K (or V) ring, from rk (rv)
    long long out_elems;      // elements of out the call may write, from out
};

// 5-D views (head dim, frame, head, token, video) of the chunk tensors; boxes of
// D x 16 frames x G heads (D x 8 x G for q).  The rings are read with 1-D bulk copies.
struct TemporalMaps {
    CUtensorMap q, k, v;
};

constexpr int kMaxRingSlots = 16 * 32;   // the ring-box mask has 32 bits

uint32_t temporal_smem_bytes(int G, int D);
cudaError_t launch_temporal(const TemporalMaps &m, const TemporalParams &p, int grid, cudaStream_t stream);

// ---- cache write ------------------------------------------------------------------------
constexpr int kMaxLayersPerWrite = 64;

struct CacheWriteLayer {
    const uint4 *kt, *vt, *ks, *vs;     // caller chunk tensors of one layer
};

struct CacheWriteParams {
    CacheWriteLayer layer[kMaxLayersPerWrite];
    uint4 *tbuf;            // temporal cache base [N_L][2][B][HW][H][Pmax][D] (token-major, head-major ring)
    uint4 *sbuf;            // spatial cache base  [N_L][2][P'][B][HW][C]
    long long row_vec;      // 16-byte vectors of this cache's C = H*D channels in a row
    long long src_row_vec;  // 16-byte vectors from one source row to the next (row pitch / 8)
    int head_vec;           // 16-byte vectors per head row of D elements
    int heads;
    long long tokens;       // B * HW
    int hw;
    int layer0;             // absolute index of layer[0]
    int n_layers;           // layers in this launch
    int n;                  // frames written
    int slot0;              // ring slot of frame 0: (head + count) mod Pmax
    int p_max;
    int n_sp;               // spatial frames written: min(P', n)
    int p_spatial;
    long long t_src_vec;    // 16-byte vectors a temporal source may be read at, from its pointer
    long long s_src_vec;    // the same for a spatial source
    long long tbuf_vec;     // 16-byte vectors of the whole temporal buffer, from tbuf
    long long sbuf_vec;     // the same for the spatial buffer
};

cudaError_t launch_cache_write(const CacheWriteParams &p, cudaStream_t stream);

// ---- prefix-enhanced spatial attention (tcgen05) -------------------------------------
struct SpatialParams {
    int B, n, H, HW, D;
    int n_src;      // key sources: own frame + spatial-cache frames
    int nkb;        // 128-key blocks per source: ceil(HW / 128)
    int q_pairs;    // pairs of 128-query tiles per frame: ceil(HW / 256)
    float scale_log2;
};

// Loaded tensors: boxes of 32 head-dims x 128 tokens with the 64-byte swizzle.
// o: boxes of D x 32 tokens, no swizzle (each softmax warp stores its 32 output rows).
struct SpatialMaps {
    CUtensorMap q, k, v, sk, sv, o;
};

uint32_t spatial_smem_bytes(int D);
cudaError_t launch_spatial(const SpatialMaps &maps, const SpatialParams &p, cudaStream_t stream);

// ---- cyclic TPE added to a chunk ------------------------------------------------------------
struct TpeAddParams {
    const uint4 *x;         // token-major chunk [B][HW][n][C] (16-byte vectors)
    uint4 *out;             // same layout; may equal x
    const uint4 *table;     // [N_tpe][C]
    long long rows;         // B * HW * n
    int row_vec;            // 16-byte vectors of the C = H*D channels added per row
    int pitch_vec;          // 16-byte vectors from one row of x, out or table to the next
    int n;                  // chunk frames
    int tpe_row[kMaxChunk]; // table row of each chunk frame
    long long xo_vec;       // 16-byte vectors of x (and of out) the call may touch
    long long table_vec;    // 16-byte vectors of the table
};

cudaError_t launch_tpe_add(const TpeAddParams &p, cudaStream_t stream);

// ---- K/V projection of the cache-writing stage, stored straight into the caches ----------
// Output tiles of 128 rows x 256 channels over [K | V] (2C channels); temporal tiles first,
// then spatial tiles.  Rows: temporal (b, s, f) of the token-major chunk input; spatial
// (s) of one of the chunk's last n_sp frames.
// Output channels per tile (TMEM columns of the accumulator) and k-steps of 64 input
// channels in flight.  Measured at C = 1152 (one layer, 2048 + 768 rows): 192 x 5 stages
// 24.9 us, 128 x 6 stages 27.9 us, 256 x 4 stages 30.4 us -- a deeper ring and 1.8 rather
// than 1.3 waves of tiles on the 148 SMs.
constexpr int kProjBN = 192;
constexpr int kProjStages = 5;

struct KvProjParams {
    __nv_bfloat16 *ring_k, *ring_v;       // this layer's K and V rings [B][HW][H][Pmax][D]
    __nv_bfloat16 *sp_k, *sp_v;           // this layer's spatial cache [P'][B][HW][H][D]
    const __nv_bfloat16 *bias_t, *bias_s; // [2C] or null
    int B, HW, H, D, C, n;
    int p_max, slot0;       // ring slot of chunk frame 0
    int n_sp;               // chunk frames stored in the spatial cache (the last n_sp)
    int rows_t;             // B * HW * n
    int tiles_n;            // ceil(2C / kProjBN)
    int tiles_t;            // temporal tiles: ceil(rows_t / 128) * tiles_n
    int tiles_s_frame;      // spatial row tiles per frame: ceil(HW / 128)
    int k_steps;            // ceil(C / 64)
    int total_tiles;        // temporal + spatial tiles (the persistent grid walks them)
    long long ring_elems;   // elements of one layer's K (or V) ring, from ring_k (ring_v)
    long long sp_elems;     // elements of one layer's spatial K (or V), from sp_k (sp_v)
};

// A tiles: boxes of 64 channels x 128 rows (x 1 frame); W tiles: 64 channels x kProjBN rows;
// all with 128-byte rows and the 128-byte swizzle.  xt, wt: 3-D views with one plane;
// xs: (channel, token, frame) of the frame-major chunk input.
struct KvProjMaps {
    CUtensorMap xt, wt, xs, ws;
};

cudaError_t launch_kv_proj(const KvProjMaps &maps, const KvProjParams &p, int grid, cudaStream_t stream);

// ---- device status word -------------------------------------------------------------------
// 0 = fine; codes below kStatusRangeCode name the bounded wait that gave up, codes from it on
// an input value outside the supported range (device code records them with record_status).
constexpr int kStatusRangeCode = 1000;
// codes from kStatusBoundsCode on: a failed bounds check of the debug build (site added)
constexpr int kStatusBoundsCode = 2000;

// ---- bounded-wait self test ---------------------------------------------------------------
cudaError_t launch_timeout_selftest(unsigned long long limit_ns, cudaStream_t stream);
int read_and_clear_status(int *status);

}  // namespace ca2
