// ca2_kernels.h -- launch interface between the C-ABI layer (ca2_api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace ca2 {

// ---- causal temporal attention ---------------------------------------------------------
constexpr int kMaxTemporalGroup = 4;   // heads per work item = consumer warps per CTA
constexpr int kMaxChunk = 8;           // queries per (token, head): the chunk length limit

struct TemporalParams {
    const __nv_bfloat16 *q, *k, *v;     // chunk tensors [B][n][HW][H][D]
    __nv_bfloat16 *out;                 // [B][n][HW][H][D]
    const __nv_bfloat16 *ring_k;        // this layer's K ring [Pmax][B][HW][H][D]
    const __nv_bfloat16 *ring_v;        // this layer's V ring
    int B, HW, H, D;
    int n;          // chunk frames in this call (queries per token-head)
    int Pk;         // queued frames
    int head;       // ring slot of the oldest queued frame
    int Pmax;
    int G;          // heads per work item
    int n_items;    // B * HW * (H / G)
    int n_stages;   // ceil((Pk + n) / 16)
    float scale_log2;   // log2(e) / sqrt(D)
    uint32_t row_bytes; // G * D * 2
    uint32_t pitch;     // shared-memory row pitch
};

uint32_t temporal_pitch(int G, int D);
uint32_t temporal_smem_bytes(int G, int D);
cudaError_t launch_temporal(const TemporalParams &p, int grid, cudaStream_t stream);

// ---- cache write ------------------------------------------------------------------------
constexpr int kMaxLayersPerWrite = 64;

struct CacheWriteLayer {
    const uint4 *kt, *vt, *ks, *vs;     // caller chunk tensors of one layer
};

struct CacheWriteParams {
    CacheWriteLayer layer[kMaxLayersPerWrite];
    uint4 *tbuf;            // temporal cache base [N_L][2][Pmax][B][plane]
    uint4 *sbuf;            // spatial cache base  [N_L][2][P'][B][plane]
    long long plane_vec;    // 16-byte vectors per (video, frame) plane: HW*H*D/8
    int layer0;             // absolute index of layer[0]
    int n_layers;           // layers in this launch
    int n;                  // frames written
    int B;
    int slot0;              // ring slot of frame 0: (head + count) mod Pmax
    int p_max;
    int n_sp;               // spatial frames written: min(P', n)
    int p_spatial;
};

cudaError_t launch_cache_write(const CacheWriteParams &p, cudaStream_t stream);

// ---- prefix-enhanced spatial attention (tcgen05) -------------------------------------
struct SpatialParams {
    int B, n, H, HW, D;
    int n_src;      // key sources: own frame + spatial-cache frames
    int nkb;        // 128-key blocks per source: ceil(HW / 128)
    int q_tiles;    // 128-query tiles per frame: ceil(HW / 128)
    float scale_log2;
};

struct SpatialMaps {
    CUtensorMap q, k, v, sk, sv, o;
};

uint32_t spatial_smem_bytes(int D);
cudaError_t launch_spatial(const SpatialMaps &maps, const SpatialParams &p, cudaStream_t stream);

// ---- bounded-wait self test ---------------------------------------------------------------
cudaError_t launch_timeout_selftest(unsigned long long limit_ns, cudaStream_t stream);
int read_and_clear_status(int *status);

}  // namespace ca2
