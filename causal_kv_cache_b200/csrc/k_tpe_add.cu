// k_tpe_add.cu -- cyclic temporal position embeddings added to a chunk (sm_100a).
//
// Ca2-VDM ("Ca2-VDM" papernotes page, 关键设计 4, "Cyclic-TPEs"): global frame g carries the
// temporal position embedding at index (offset + g) mod N_tpe; once the table runs out the
// indices start again from the beginning.  This kernel adds, to every token's C = H*D vector
// of frame f of a chunk, the table row of that frame's index: the temporal branch's input
// plus its cyclic TPE.  The indices are computed on the host and passed by value.
//
// HBM-bound elementwise work: each 16-byte vector of the chunk is read once and written
// once; the n table rows (n * C * 2 bytes) stay in L1/L2.  Each element is the float32 sum
// of the two bf16 values rounded once to bf16 (nearest, ties to even).  Plain loads (not the
// read-only path), so the output may alias the input.
#include <cstdint>

#include "ca2_device.cuh"
#include "ca2_kernels.h"

namespace ca2 {

namespace {
constexpr int kThreads = 256;
constexpr int kVecPerThread = 4;

// eight bf16 lanes of x plus eight of t, each sum rounded once to bf16
__device__ __forceinline__ uint4 add8(const uint4 &x, const uint4 &t)
{
    auto add2 = [](uint32_t a, uint32_t b) {
        return pack_bf16x2(bf16_lo(a) + bf16_lo(b), bf16_hi(a) + bf16_hi(b));
    };
    return make_uint4(add2(x.x, t.x), add2(x.y, t.y), add2(x.z, t.z), add2(x.w, t.w));
}
}  // namespace

__global__ void __launch_bounds__(kThreads) k_tpe_add(const TpeAddParams p)
{
    // the chunk is produced by the previous kernel on the stream
    wait_previous_kernel();
    allow_next_kernel();
    // 32-bit index arithmetic: the host guarantees rows * pitch_vec < 2^31
    const uint32_t total = (uint32_t)(p.rows * (long long)p.row_vec);
    const uint32_t rv = (uint32_t)p.row_vec, pv = (uint32_t)p.pitch_vec, n = (uint32_t)p.n;
    const uint32_t base = blockIdx.x * (uint32_t)(kThreads * kVecPerThread) + threadIdx.x;
    uint4 xv[kVecPerThread], tv[kVecPerThread];
    uint32_t xi[kVecPerThread];
#pragma unroll
    for (int i = 0; i < kVecPerThread; ++i) {
        const uint32_t e = base + (uint32_t)(i * kThreads);
        if (e < total) {
            const uint32_t row = e / rv;                    // (video, token, frame) row
            const uint32_t v = e - row * rv;                // 16-byte vector within the row
            const uint32_t f = row % n;                     // chunk frame (token-major rows)
            xi[i] = row * pv + v;
            const uint32_t ti = (uint32_t)p.tpe_row[f] * pv + v;
            xv[i] = CA2_IN_BOUNDS(xi[i] < p.xo_vec, 51) ? p.x[xi[i]] : make_uint4(0u, 0u, 0u, 0u);
            tv[i] = CA2_IN_BOUNDS(ti < p.table_vec, 52) ? p.table[ti] : make_uint4(0u, 0u, 0u, 0u);
        }
    }
#pragma unroll
    for (int i = 0; i < kVecPerThread; ++i) {
        const uint32_t e = base + (uint32_t)(i * kThreads);
        if (e < total && CA2_IN_BOUNDS(xi[i] < p.xo_vec, 53)) p.out[xi[i]] = add8(xv[i], tv[i]);
    }
}

cudaError_t launch_tpe_add(const TpeAddParams &p, cudaStream_t stream)
{
    const long long per_block = (long long)kThreads * kVecPerThread;
    const long long total = p.rows * (long long)p.row_vec;
    if (total == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((total + per_block - 1) / per_block);
    return launch_chained(k_tpe_add, dim3(grid), dim3(kThreads), 0, stream, p);
}

}  // namespace ca2
