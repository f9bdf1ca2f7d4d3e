// ca2_api.cu -- the extern "C" surface of libca2.so (declared in include/ca2.h).
//
// Host side of the Ca2-VDM cached attention path: argument validation, the ring-buffer
// state of the temporal KV-cache queue (head / count kept on the host and passed to the
// kernels by value), the spatial-cache frame count, cyclic TPE indices, tensor-map
// encoding for the tensor-core kernel, and kernel launches on the caller's stream.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "ca2.h"
#include "ca2_kernels.h"

struct ca2_cache {
    ca2_config cfg;
    uint8_t *tbuf;      // [N_L][2][B][HW][H][Pmax][D] bf16 (token-major, head-major ring)
    uint8_t *sbuf;      // [N_L][2][P'][B][HW][H][D] bf16
    size_t plane_bytes; // bytes of one frame-plane B*HW*H*D*2
    int head;           // ring slot of the oldest queued frame
    int count;          // queued frames
    int sp_count;       // frames in the spatial cache
    long long frames_written;
};

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate_config(const ca2_config *c)
{
    if (!c) return CA2_ERR_ARG;
    if (c->n_layers < 1 || c->batch < 1 || c->hw < 1 || c->heads < 1) return CA2_ERR_SHAPE;
    if (c->head_dim < 8 || c->head_dim > 128 || (c->head_dim % 8) != 0) return CA2_ERR_SHAPE;
    if (c->chunk_len < 1 || c->chunk_len > ca2::kMaxChunk) return CA2_ERR_SHAPE;
    if (c->p_max < c->chunk_len || c->p_max > ca2::kMaxRingSlots) return CA2_ERR_SHAPE;
    if (c->p_spatial < 0 || c->p_spatial > c->chunk_len) return CA2_ERR_SHAPE;
    if (c->tpe_len < 0) return CA2_ERR_SHAPE;
    // tensor-map extents and 32-bit strides
    const long long hd = (long long)c->heads * c->head_dim;
    if (hd * c->hw * 2 > (1ll << 40) || c->hw > (1 << 30)) return CA2_ERR_SHAPE;
    // rows of the caller's chunk tensors: 16-byte multiples, at least this cache's heads
    if (c->row_pitch != 0 && (c->row_pitch < hd || (c->row_pitch % 8) != 0 || c->row_pitch > (1 << 24)))
        return CA2_ERR_SHAPE;
    const long long pitch = c->row_pitch ? c->row_pitch : hd;
    if (pitch * c->hw * c->chunk_len * 2 > (1ll << 40)) return CA2_ERR_SHAPE;
    return CA2_OK;
}

size_t plane_bytes_of(const ca2_config *c)
{
    return (size_t)c->batch * (size_t)c->hw * (size_t)c->heads * (size_t)c->head_dim * 2u;
}

// Name of the last CUDA error a call of this library met (per host thread).
thread_local const char *g_last_cuda_error = "no error";

int cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return CA2_OK;
    g_last_cuda_error = cudaGetErrorString(e);
    return CA2_ERR_CUDA;
}

// Multiprocessor count of the current device, read once per device (devices past 63 are
// queried on every call).
int sm_count()
{
    static std::atomic<int> cached[64];   // 0 = not read yet
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) {
        const int n = cached[dev].load(std::memory_order_relaxed);
        if (n > 0) return n;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

// The driver's tensor-map encoder, looked up once (thread-safe static initialisation).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        return nullptr;
    }();
    return fn;
}

// View a bf16 tensor [frames][HW][H][D] whose token rows are `pitch` elements apart as 4-D
// (D, H, HW, frames) and encode a tiled map.
bool encode_4d(CUtensorMap *m, const void *base, int D, int H, int HW, int frames, long long pitch, int box_d,
               int box_rows, CUtensorMapSwizzle swz)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)HW, (cuuint64_t)frames};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)pitch * 2, (cuuint64_t)HW * pitch * 2};
    cuuint32_t box[4] = {(cuuint32_t)box_d, 1u, (cuuint32_t)box_rows, 1u};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 5-D view (D, frames, H, HW, B) of a bf16 tensor with the given frame, token and video
// strides (elements; heads are D apart); box D x box_frames x box_heads x 1 x 1, no swizzle.
bool encode_5d(CUtensorMap *m, const void *base, int D, int frames, int H, int HW, int B, long long frame_stride,
               long long token_stride, long long video_stride, int box_frames, int box_heads)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)frames, (cuuint64_t)H, (cuuint64_t)HW, (cuuint64_t)B};
    cuuint64_t strides[4] = {(cuuint64_t)frame_stride * 2, (cuuint64_t)D * 2, (cuuint64_t)token_stride * 2,
                             (cuuint64_t)video_stride * 2};
    cuuint32_t box[5] = {(cuuint32_t)D, (cuuint32_t)box_frames, (cuuint32_t)box_heads, 1u, 1u};
    cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D view (channel, row, plane) of a bf16 matrix stack with the given row and plane
// strides (elements); box 64 channels x box_rows x 1, 128-byte swizzle (GEMM operand tiles).
bool encode_rows_3d(CUtensorMap *m, const void *base, long long cols, long long rows, long long planes,
                    long long row_stride, long long plane_stride, int box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)planes};
    cuuint64_t strides[2] = {(cuuint64_t)row_stride * 2, (cuuint64_t)plane_stride * 2};
    cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

uint8_t *layer_ring(const ca2_cache *c, int layer, int kv)
{
    return c->tbuf + ((size_t)layer * 2 + (size_t)kv) * (size_t)c->cfg.p_max * c->plane_bytes;
}

uint8_t *layer_spatial(const ca2_cache *c, int layer, int kv)
{
    return c->sbuf + ((size_t)layer * 2 + (size_t)kv) * (size_t)c->cfg.p_spatial * c->plane_bytes;
}

int check_chunk_args(const ca2_cache *c, int layer, const void *q, const void *k, const void *v, const void *out,
                     int n)
{
    if (!c || !q || !k || !v || !out) return CA2_ERR_ARG;
    if (layer < 0 || layer >= c->cfg.n_layers) return CA2_ERR_ARG;
    if (n < 1 || n > c->cfg.chunk_len) return CA2_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return CA2_ERR_ALIGN;
    return CA2_OK;
}

}  // namespace

extern "C" {

int ca2_cache_bytes(const ca2_config *cfg, size_t *temporal_bytes, size_t *spatial_bytes)
{
    int st = validate_config(cfg);
    if (st != CA2_OK) return st;
    const size_t plane = plane_bytes_of(cfg);
    if (temporal_bytes) *temporal_bytes = 2u * (size_t)cfg->n_layers * (size_t)cfg->p_max * plane;
    if (spatial_bytes) *spatial_bytes = 2u * (size_t)cfg->n_layers * (size_t)cfg->p_spatial * plane;
    return CA2_OK;
}

int ca2_cache_init(const ca2_config *cfg, void *temporal_buf, size_t temporal_bytes, void *spatial_buf,
                   size_t spatial_bytes, ca2_cache **out)
{
    if (!out) return CA2_ERR_ARG;
    *out = nullptr;
    int st = validate_config(cfg);
    if (st != CA2_OK) return st;
    size_t need_t = 0, need_s = 0;
    ca2_cache_bytes(cfg, &need_t, &need_s);
    if (!temporal_buf) return CA2_ERR_ARG;
    if (need_s > 0 && !spatial_buf) return CA2_ERR_ARG;
    if (temporal_bytes < need_t || spatial_bytes < need_s) return CA2_ERR_CAPACITY;
    if (!aligned16(temporal_buf) || (spatial_buf && !aligned16(spatial_buf))) return CA2_ERR_ALIGN;
    ca2_cache *c = new (std::nothrow) ca2_cache;
    if (!c) return CA2_ERR_ARG;
    c->cfg = *cfg;
    if (c->cfg.tpe_len == 0) c->cfg.tpe_len = cfg->p_max + cfg->chunk_len;
    if (c->cfg.row_pitch == 0) c->cfg.row_pitch = cfg->heads * cfg->head_dim;
    c->tbuf = static_cast<uint8_t *>(temporal_buf);
    c->sbuf = static_cast<uint8_t *>(spatial_buf);
    c->plane_bytes = plane_bytes_of(cfg);
    c->head = 0;
    c->count = 0;
    c->sp_count = 0;
    c->frames_written = 0;
    *out = c;
    return CA2_OK;
}

int ca2_cache_destroy(ca2_cache *cache)
{
    delete cache;
    return CA2_OK;
}

int ca2_cache_config(const ca2_cache *c, ca2_config *out)
{
    if (!c || !out) return CA2_ERR_ARG;
    *out = c->cfg;
    return CA2_OK;
}

int ca2_cache_layer_offsets(const ca2_cache *c, int layer, int kv, size_t *temporal_offset, size_t *spatial_offset)
{
    if (!c || layer < 0 || layer >= c->cfg.n_layers || (kv != 0 && kv != 1)) return CA2_ERR_ARG;
    if (temporal_offset) *temporal_offset = (size_t)(layer_ring(c, layer, kv) - c->tbuf);
    if (spatial_offset)
        *spatial_offset = ((size_t)layer * 2 + (size_t)kv) * (size_t)c->cfg.p_spatial * c->plane_bytes;
    return CA2_OK;
}

int ca2_cache_evict(ca2_cache *c, int n)
{
    if (!c) return CA2_ERR_ARG;
    if (n < 0 || n > c->count) return CA2_ERR_CAPACITY;
    c->head = (c->head + n) % c->cfg.p_max;
    c->count -= n;
    return CA2_OK;
}

int ca2_cache_evict_for(ca2_cache *c, int n_new, int *evicted)
{
    if (!c) return CA2_ERR_ARG;
    if (n_new < 0 || n_new > c->cfg.p_max) return CA2_ERR_SHAPE;
    const int e = c->count + n_new > c->cfg.p_max ? c->count + n_new - c->cfg.p_max : 0;
    const int st = ca2_cache_evict(c, e);
    if (st != CA2_OK) return st;
    if (evicted) *evicted = e;
    return CA2_OK;
}

int ca2_cache_write(ca2_cache *c, const void *const *k_t, const void *const *v_t, const void *const *k_s,
                    const void *const *v_s, int n, void *stream)
{
    if (!c || !k_t || !v_t) return CA2_ERR_ARG;
    const ca2_config &g = c->cfg;
    if (n < 1 || n > g.chunk_len) return CA2_ERR_SHAPE;
    if (c->count + n > g.p_max) return CA2_ERR_CAPACITY;
    const int n_sp = n < g.p_spatial ? n : g.p_spatial;
    if (n_sp > 0 && (!k_s || !v_s)) return CA2_ERR_ARG;
    for (int L = 0; L < g.n_layers; ++L) {
        if (!k_t[L] || !v_t[L]) return CA2_ERR_ARG;
        if (!aligned16(k_t[L]) || !aligned16(v_t[L])) return CA2_ERR_ALIGN;
        if (n_sp > 0) {
            if (!k_s[L] || !v_s[L]) return CA2_ERR_ARG;
            if (!aligned16(k_s[L]) || !aligned16(v_s[L])) return CA2_ERR_ALIGN;
        }
    }
    ca2::CacheWriteParams p;
    std::memset(&p, 0, sizeof(p));
    p.tbuf = reinterpret_cast<uint4 *>(c->tbuf);
    p.sbuf = reinterpret_cast<uint4 *>(c->sbuf);
    p.row_vec = (long long)g.heads * g.head_dim / 8;   // 16-byte vectors of this cache's heads per row
    p.src_row_vec = (long long)g.row_pitch / 8;        // 16-byte vectors from one source row to the next
    p.tokens = (long long)g.batch * g.hw;
    p.head_vec = g.head_dim / 8;                       // 16-byte vectors per head row
    p.heads = g.heads;
    p.hw = g.hw;
    p.n = n;
    p.slot0 = (c->head + c->count) % g.p_max;
    p.p_max = g.p_max;
    p.n_sp = n_sp;
    p.p_spatial = g.p_spatial;
    // extents for the debug build's bounds checks
    p.t_src_vec = (p.tokens * n - 1) * p.src_row_vec + p.row_vec;
    p.s_src_vec = ((long long)g.batch * n * g.hw - 1) * p.src_row_vec + p.row_vec;
    p.tbuf_vec = (long long)g.n_layers * 2 * p.tokens * g.p_max * p.row_vec;
    p.sbuf_vec = (long long)g.n_layers * 2 * g.p_spatial * p.tokens * p.row_vec;
    for (int L0 = 0; L0 < g.n_layers; L0 += ca2::kMaxLayersPerWrite) {
        const int nl = (g.n_layers - L0) < ca2::kMaxLayersPerWrite ? (g.n_layers - L0) : ca2::kMaxLayersPerWrite;
        p.layer0 = L0;
        p.n_layers = nl;
        for (int i = 0; i < nl; ++i) {
            p.layer[i].kt = static_cast<const uint4 *>(k_t[L0 + i]);
            p.layer[i].vt = static_cast<const uint4 *>(v_t[L0 + i]);
            p.layer[i].ks = n_sp > 0 ? static_cast<const uint4 *>(k_s[L0 + i]) : nullptr;
            p.layer[i].vs = n_sp > 0 ? static_cast<const uint4 *>(v_s[L0 + i]) : nullptr;
        }
        const int st = cuda_status(ca2::launch_cache_write(p, static_cast<cudaStream_t>(stream)));
        if (st != CA2_OK) return st;
    }
    c->count += n;
    c->sp_count = n_sp;
    c->frames_written += n;
    return CA2_OK;
}

int ca2_temporal_attn(ca2_cache *c, int layer, const void *q, const void *k, const void *v, void *out, int n,
                      void *stream)
{
    int st = check_chunk_args(c, layer, q, k, v, out, n);
    if (st != CA2_OK) return st;
    const ca2_config &g = c->cfg;
    ca2::TemporalParams p;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.B = g.batch;
    p.HW = g.hw;
    p.H = g.heads;
    p.D = g.head_dim;
    p.n = n;
    p.Pk = c->count;
    p.head = c->head;
    p.Pmax = g.p_max;
    int G = ca2::kMaxTemporalGroup;
    while (g.heads % G) G >>= 1;
    p.G = G;
    p.n_items = g.batch * g.hw * (g.heads / G);
    p.ring_box_mask = 0;
    for (int i = 0; i < c->count; ++i) p.ring_box_mask |= 1u << (((c->head + i) % g.p_max) / 16);
    p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)g.head_dim));
    p.ring_bytes = (long long)g.batch * g.hw * g.heads * g.p_max * g.head_dim * 2;
    p.out_elems = ((long long)g.batch * g.hw * n - 1) * g.row_pitch + (long long)g.heads * g.head_dim;

    // temporal chunk tensors are token-major [B][HW][n][H][D] (C = H*D), read as TMA boxes;
    // the ring [B][HW][H][Pmax][D] is read with bulk copies of one head's consecutive slots
    const long long C = g.row_pitch;                   // elements from one chunk row to the next
    p.pitch = g.row_pitch;
    p.rk = layer_ring(c, layer, 0);
    p.rv = layer_ring(c, layer, 1);
    ca2::TemporalMaps m;
    const bool ok =
        encode_5d(&m.q, q, g.head_dim, n, g.heads, g.hw, g.batch, C, n * C, (long long)g.hw * n * C, 8, G) &&
        encode_5d(&m.k, k, g.head_dim, n, g.heads, g.hw, g.batch, C, n * C, (long long)g.hw * n * C, 16, G) &&
        encode_5d(&m.v, v, g.head_dim, n, g.heads, g.hw, g.batch, C, n * C, (long long)g.hw * n * C, 16, G);
    if (!ok) {
        g_last_cuda_error = "tensor-map encoding failed";
        return CA2_ERR_CUDA;
    }
    // one CTA per work item; the resident CTAs take over the items of CTAs that have not
    // started (cluster launch control), so the grid's size only fixes the work list
    const int grid = p.n_items;
    return cuda_status(ca2::launch_temporal(m, p, grid, static_cast<cudaStream_t>(stream)));
}

int ca2_spatial_prefix_attn(ca2_cache *c, int layer, const void *q, const void *k, const void *v, void *out,
                            int n, int use_prefix, void *stream)
{
    int st = check_chunk_args(c, layer, q, k, v, out, n);
    if (st != CA2_OK) return st;
    if (use_prefix != 0 && use_prefix != 1) return CA2_ERR_ARG;
    const ca2_config &g = c->cfg;
    const int n_sp = use_prefix ? c->sp_count : 0;
    const int frames = g.batch * n;
    ca2::SpatialMaps m;
    const int D = g.head_dim, H = g.heads, HW = g.hw;
    // the caller's chunk rows are row_pitch apart; the spatial cache's rows are H*D apart
    auto load_map = [&](CUtensorMap *mm, const void *base, int frames_, long long pitch) {
        return encode_4d(mm, base, D, H, HW, frames_, pitch, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B);
    };
    const long long cp = g.row_pitch, hd = (long long)H * D;
    bool ok = load_map(&m.q, q, frames, cp) && load_map(&m.k, k, frames, cp) && load_map(&m.v, v, frames, cp) &&
              encode_4d(&m.o, out, D, H, HW, frames, cp, D, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok && n_sp > 0) {
        ok = load_map(&m.sk, layer_spatial(c, layer, 0), n_sp * g.batch, hd) &&
             load_map(&m.sv, layer_spatial(c, layer, 1), n_sp * g.batch, hd);
    } else if (ok) {
        m.sk = m.k;   // never read when there is no prefix
        m.sv = m.v;
    }
    if (!ok) {
        g_last_cuda_error = "tensor-map encoding failed";
        return CA2_ERR_CUDA;
    }
    ca2::SpatialParams p;
    p.B = g.batch;
    p.n = n;
    p.H = g.heads;
    p.HW = g.hw;
    p.D = g.head_dim;
    p.n_src = 1 + n_sp;
    p.nkb = (g.hw + 127) / 128;
    p.q_pairs = (g.hw + 255) / 256;
    p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)g.head_dim));
    return cuda_status(ca2::launch_spatial(m, p, static_cast<cudaStream_t>(stream)));
}

int ca2_kv_proj_write(ca2_cache *c, int layer, const void *x_t, const void *w_t, const void *b_t, const void *x_s,
                      const void *w_s, const void *b_s, int n, void *stream)
{
    if (!c || !x_t || !w_t) return CA2_ERR_ARG;
    const ca2_config &g = c->cfg;
    if (layer < 0 || layer >= g.n_layers) return CA2_ERR_ARG;
    if (n < 1 || n > g.chunk_len) return CA2_ERR_SHAPE;
    if (c->count + n > g.p_max) return CA2_ERR_CAPACITY;
    const int n_sp = n < g.p_spatial ? n : g.p_spatial;
    if (n_sp > 0 && (!x_s || !w_s)) return CA2_ERR_ARG;
    const void *ptrs[6] = {x_t, w_t, b_t, n_sp > 0 ? x_s : nullptr, n_sp > 0 ? w_s : nullptr, n_sp > 0 ? b_s : nullptr};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return CA2_ERR_ALIGN;
    const long long C = (long long)g.heads * g.head_dim;   // output channels of K (and of V)
    const long long Cin = g.row_pitch;                       // input channels: a whole row
    const long long rows_t = (long long)g.batch * g.hw * n;
    if (rows_t >= (1ll << 31) || C * 2 >= (1ll << 31)) return CA2_ERR_SHAPE;

    ca2::KvProjParams p;
    std::memset(&p, 0, sizeof(p));
    p.ring_k = reinterpret_cast<__nv_bfloat16 *>(layer_ring(c, layer, 0));
    p.ring_v = reinterpret_cast<__nv_bfloat16 *>(layer_ring(c, layer, 1));
    p.sp_k = n_sp > 0 ? reinterpret_cast<__nv_bfloat16 *>(layer_spatial(c, layer, 0)) : nullptr;
    p.sp_v = n_sp > 0 ? reinterpret_cast<__nv_bfloat16 *>(layer_spatial(c, layer, 1)) : nullptr;
    p.bias_t = static_cast<const __nv_bfloat16 *>(b_t);
    p.bias_s = n_sp > 0 ? static_cast<const __nv_bfloat16 *>(b_s) : nullptr;
    p.B = g.batch;
    p.HW = g.hw;
    p.H = g.heads;
    p.D = g.head_dim;
    p.C = (int)C;
    p.n = n;
    p.p_max = g.p_max;
    p.slot0 = (c->head + c->count) % g.p_max;
    p.n_sp = n_sp;
    p.rows_t = (int)rows_t;
    p.tiles_n = (int)((2 * C + ca2::kProjBN - 1) / ca2::kProjBN);
    p.tiles_t = (int)((rows_t + 127) / 128) * p.tiles_n;
    p.tiles_s_frame = (g.hw + 127) / 128;
    p.k_steps = (int)((Cin + 63) / 64);
    const long long tiles_s = (long long)g.batch * n_sp * p.tiles_s_frame * p.tiles_n;
    if (p.tiles_t + tiles_s >= (1ll << 31)) return CA2_ERR_SHAPE;
    p.total_tiles = (int)(p.tiles_t + tiles_s);
    p.ring_elems = (long long)g.batch * g.hw * g.heads * g.p_max * g.head_dim;
    p.sp_elems = (long long)g.p_spatial * g.batch * g.hw * g.heads * g.head_dim;

    // x_t: [B*HW*n][Cin]; x_s: (Cin, HW, B*n frames); W: [2C][Cin] (output channel rows)
    ca2::KvProjMaps m;
    std::memset(&m, 0, sizeof(m));
    bool ok = encode_rows_3d(&m.xt, x_t, Cin, rows_t, 1, Cin, rows_t * Cin, 128) &&
              encode_rows_3d(&m.wt, w_t, Cin, 2 * C, 1, Cin, 2 * C * Cin, ca2::kProjBN);
    if (ok && n_sp > 0)
        ok = encode_rows_3d(&m.xs, x_s, Cin, g.hw, (long long)g.batch * n, Cin, (long long)g.hw * Cin, 128) &&
             encode_rows_3d(&m.ws, w_s, Cin, 2 * C, 1, Cin, 2 * C * Cin, ca2::kProjBN);
    else
        m.xs = m.xt, m.ws = m.wt;    // no spatial tile reads them
    if (!ok) {
        g_last_cuda_error = "tensor-map encoding failed";
        return CA2_ERR_CUDA;
    }
    // persistent: one CTA per SM (or per tile when there are fewer tiles)
    const int sms = sm_count();
    if (sms <= 0) return CA2_ERR_CUDA;
    const int grid = p.total_tiles < sms ? p.total_tiles : sms;
    return cuda_status(ca2::launch_kv_proj(m, p, grid, static_cast<cudaStream_t>(stream)));
}

int ca2_cache_commit(ca2_cache *c, int n)
{
    if (!c) return CA2_ERR_ARG;
    const ca2_config &g = c->cfg;
    if (n < 1 || n > g.chunk_len) return CA2_ERR_SHAPE;
    if (c->count + n > g.p_max) return CA2_ERR_CAPACITY;
    c->count += n;
    c->sp_count = n < g.p_spatial ? n : g.p_spatial;
    c->frames_written += n;
    return CA2_OK;
}

int ca2_tpe_add(const ca2_cache *c, long long first_global_frame, int offset, const void *table, const void *x,
                void *out, int n, void *stream)
{
    if (!c || !table || !x || !out) return CA2_ERR_ARG;
    if (first_global_frame < 0 || offset < 0) return CA2_ERR_ARG;
    if (n < 1 || n > c->cfg.chunk_len) return CA2_ERR_SHAPE;
    if (!aligned16(table) || !aligned16(x) || !aligned16(out)) return CA2_ERR_ALIGN;
    const ca2_config &g = c->cfg;
    const long long n_tpe = g.tpe_len;
    ca2::TpeAddParams p;
    p.x = static_cast<const uint4 *>(x);
    p.out = static_cast<uint4 *>(out);
    p.table = static_cast<const uint4 *>(table);
    p.rows = (long long)g.batch * g.hw * n;
    p.row_vec = g.heads * g.head_dim / 8;
    p.pitch_vec = g.row_pitch / 8;
    p.n = n;
    // the kernel indexes in 32 bits
    if (p.rows * p.pitch_vec >= (1ll << 31) || (long long)n_tpe * p.pitch_vec >= (1ll << 31)) return CA2_ERR_SHAPE;
    for (int i = 0; i < ca2::kMaxChunk; ++i)
        p.tpe_row[i] = i < n ? (int)(((long long)offset + first_global_frame + i) % n_tpe) : 0;
    p.xo_vec = (p.rows - 1) * p.pitch_vec + p.row_vec;
    p.table_vec = (n_tpe - 1) * p.pitch_vec + p.row_vec;
    return cuda_status(ca2::launch_tpe_add(p, static_cast<cudaStream_t>(stream)));
}

int ca2_tpe_indices(const ca2_cache *c, long long first_global_frame, int offset, int n, int *out_host)
{
    if (!c) return CA2_ERR_ARG;
    if (n < 0 || first_global_frame < 0 || offset < 0) return CA2_ERR_ARG;
    if (n > 0 && !out_host) return CA2_ERR_ARG;
    const long long N = c->cfg.tpe_len;
    for (int i = 0; i < n; ++i) out_host[i] = (int)(((long long)offset + first_global_frame + i) % N);
    return CA2_OK;
}

int ca2_cache_state(const ca2_cache *c, int *head, int *count, int *sp_count, long long *frames_written)
{
    if (!c) return CA2_ERR_ARG;
    if (head) *head = c->head;
    if (count) *count = c->count;
    if (sp_count) *sp_count = c->sp_count;
    if (frames_written) *frames_written = c->frames_written;
    return CA2_OK;
}

int ca2_device_status(void)
{
    if (cudaDeviceSynchronize() != cudaSuccess) return CA2_ERR_CUDA;
    int s = 0;
    if (ca2::read_and_clear_status(&s) != 0) return CA2_ERR_CUDA;
    if (s == 0) return CA2_OK;
    if (s >= ca2::kStatusBoundsCode) return CA2_ERR_BOUNDS;
    return s >= ca2::kStatusRangeCode ? CA2_ERR_RANGE : CA2_ERR_TIMEOUT;
}

int ca2_selftest_timeout(int wait_us, void *stream)
{
    if (wait_us < 1 || wait_us > 1000000) return CA2_ERR_ARG;
    return cuda_status(
        ca2::launch_timeout_selftest((unsigned long long)wait_us * 1000ull, static_cast<cudaStream_t>(stream)));
}

int ca2_head_shard(int heads, int world, int rank, int *h0, int *h_count)
{
    if (world < 1 || heads < world || rank < 0 || rank >= world) return CA2_ERR_SHAPE;
    const int base = heads / world, extra = heads % world;
    if (h0) *h0 = rank * base + (rank < extra ? rank : extra);
    if (h_count) *h_count = base + (rank < extra ? 1 : 0);
    return CA2_OK;
}

int ca2_debug_build(void)
{
#ifdef CA2_DEBUG
    return 1;
#else
    return 0;
#endif
}

const char *ca2_last_error_string(void) { return g_last_cuda_error; }

const char *ca2_status_string(int s)
{
    switch (s) {
    case CA2_OK: return "ok";
    case CA2_ERR_ARG: return "invalid argument";
    case CA2_ERR_SHAPE: return "size outside the supported range";
    case CA2_ERR_CAPACITY: return "capacity exceeded";
    case CA2_ERR_ALIGN: return "pointer not 16-byte aligned";
    case CA2_ERR_CUDA: return "CUDA runtime error";
    case CA2_ERR_TIMEOUT: return "device wait timed out";
    case CA2_ERR_RANGE: return "input value outside the supported range";
    case CA2_ERR_BOUNDS: return "bounds check failed (debug build)";
    default: return "unknown status";
    }
}

}  // extern "C"
