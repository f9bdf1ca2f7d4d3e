// k_temporal.cu -- causal temporal attention over the cached prefix queue (sm_100a).
//
// Ca2-VDM ("Ca2-VDM" papernotes page, 关键设计 1, equation CausalAttn): per spatial token
// and head, the l queries of the current chunk attend to the P_k queued clean-prefix
// frames (oldest first) followed by the chunk's own frames 0..c, i.e. the rows of
// Softmax(QK^T/sqrt(D) + M)V that belong to the chunk, with M_ij = -inf for i < j.
//
// Design (HBM-bound: every cached K/V byte is read once per call):
//   * Work item = (video b, token s, group of G heads).  The G*D*2-byte run of one frame
//     at (b, s, heads of the group) is contiguous in both the chunk tensors and the ring
//     slots, so each key frame arrives with one 1-D bulk copy (TMA engine).
//   * Persistent CTAs: one producer warp streams items' key frames through an NS-deep
//     ring of 16-frame stages (K and V), completing on mbarriers; G consumer warps (one
//     head each) compute.  The producer runs ahead into the next item, so loads stay in
//     flight across item boundaries.
//   * Per head the contraction is tiny (8 queries x <=16 keys per stage x D), so both
//     products use mma.sync on registers: S^T = K Q^T (keys on the M axis, queries on
//     N = 8, no padding of the query axis), then O^T += V^T P^T.  Each lane owns the
//     same two query columns in both accumulators, so the online-softmax rescale is
//     lane-local; P^T is turned into the B operand with movmatrix.  The causal mask and
//     the queue-length mask are applied to the scores in registers.
//   * Output rows are transposed back with movmatrix and stored by each lane.
#include <cstdint>
#include <cuda_bf16.h>

#include "ca2_device.cuh"
#include "ca2_kernels.h"

namespace ca2 {

namespace {

constexpr int kStages = 4;      // key stages in flight per CTA
constexpr int kKeysPerStage = 16;
constexpr int kQTile = 8;       // queries per head (chunk frames), the mma N extent

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x1(uint32_t addr, uint32_t &r0)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x1.shared.b16 {%0}, [%1];" : "=r"(r0) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t &r0, uint32_t &r1)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ uint32_t movm_t(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma1688(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0)
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(b0));
}
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct Layout {
    uint32_t stage_bytes;   // K rows then V rows of one stage
    uint32_t q_off, bar_off, total;
};

__host__ __device__ inline Layout make_layout(uint32_t pitch)
{
    Layout L;
    L.stage_bytes = 2u * kKeysPerStage * pitch;
    L.q_off = kStages * L.stage_bytes;
    L.bar_off = L.q_off + 2u * kQTile * pitch;
    L.total = L.bar_off + 8u * (2 * kStages + 4) + 16u;
    return L;
}

}  // namespace

template <int DT>
__global__ void __launch_bounds__(32 * (kMaxTemporalGroup + 1)) k_temporal_causal(const TemporalParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = p.G;
    const uint32_t pitch = p.pitch;
    const Layout L = make_layout(pitch);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L.bar_off;
    auto full_bar = [&](int i) { return bar0 + 8u * i; };
    auto empty_bar = [&](int i) { return bar0 + 8u * (kStages + i); };
    auto qfull_bar = [&](int i) { return bar0 + 8u * (2 * kStages + i); };
    auto qempty_bar = [&](int i) { return bar0 + 8u * (2 * kStages + 2 + i); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.bar_off + 8u * (2 * kStages + 4));

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(full_bar(i), 1);
            mbar_init(empty_bar(i), G);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(qfull_bar(i), 1);
            mbar_init(qempty_bar(i), G);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const int HD = p.H * p.D;                      // elements per token
    const int groups = p.H / G;
    const int nk = p.Pk + p.n;                     // keys per query row, before the mask
    const long long plane = (long long)p.B * p.HW * HD;
    const uint32_t rb = p.row_bytes;

    if (warp == G) {
        // ------------------------------ producer ------------------------------------
        int stage = 0, li = 0;
        bool ok = true;
        for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++li) {
            const int hg = it % groups;
            const int s = (it / groups) % p.HW;
            const int b = it / (groups * p.HW);
            const long long tok = ((long long)b * p.HW + s) * HD + (long long)hg * G * p.D;   // in a frame-plane
            const int qs = li & 1;
            if (li >= 2 && !mbar_wait(qempty_bar(qs), ((li - 2) >> 1) & 1, 101, abort_flag)) { ok = false; break; }
            if (lane == 0) mbar_expect_tx(qfull_bar(qs), (uint32_t)p.n * rb);
            __syncwarp();
            if (lane < p.n) {
                const __nv_bfloat16 *src = p.q + (((long long)b * p.n + lane) * p.HW + s) * HD + (long long)hg * G * p.D;
                bulk_g2s(sbase + L.q_off + (uint32_t)(qs * kQTile + lane) * pitch, src, rb, qfull_bar(qs));
            }
            for (int st = 0; st < p.n_stages; ++st, ++stage) {
                const int slot = stage % kStages;
                if (stage >= kStages &&
                    !mbar_wait(empty_bar(slot), ((stage / kStages) - 1) & 1, 102, abort_flag)) { ok = false; break; }
                if (lane == 0) mbar_expect_tx(full_bar(slot), 2u * kKeysPerStage * rb);
                __syncwarp();
                // lanes 0..15 copy K rows, lanes 16..31 the V rows of the same key frames
                const int r = lane & 15;
                int kf = st * kKeysPerStage + r;
                if (kf > nk - 1) kf = nk - 1;          // pad with a real (finite) frame; masked later
                const bool is_v = lane >= 16;
                const __nv_bfloat16 *src;
                if (kf < p.Pk) {
                    int slot_r = p.head + kf;
                    if (slot_r >= p.Pmax) slot_r -= p.Pmax;
                    src = (is_v ? p.ring_v : p.ring_k) + (long long)slot_r * plane + tok;
                } else {
                    const int c = kf - p.Pk;
                    src = (is_v ? p.v : p.k) + (((long long)b * p.n + c) * p.HW + s) * HD + (long long)hg * G * p.D;
                }
                const uint32_t dst = sbase + (uint32_t)slot * L.stage_bytes + (uint32_t)((is_v ? kKeysPerStage : 0) + r) * pitch;
                bulk_g2s(dst, src, rb, full_bar(slot));
            }
        }
        // Drain: make sure no copy issued by this CTA is still landing when it exits.
        if (!ok) {
            for (int i = 0; i < kStages; ++i) mbar_wait(full_bar(i), 0, 0, nullptr, 1000000ull);
        }
    } else if (warp < G) {
        // ------------------------------ consumers -----------------------------------
        const int w = warp;
        const uint32_t head_off = (uint32_t)(w * p.D * 2);
        int stage = 0, li = 0;
        const int q0 = 2 * (lane & 3);           // this lane's two query columns: q0, q0 + 1
        const int krow = lane >> 2;               // this lane's key rows: krow, krow + 8
        const float kNegInf = __int_as_float(0xff800000);
        for (int it = blockIdx.x; it < p.n_items; it += gridDim.x, ++li) {
            const int hg = it % groups;
            const int s = (it / groups) % p.HW;
            const int b = it / (groups * p.HW);
            const int qs = li & 1;
            if (!mbar_wait(qfull_bar(qs), (li >> 1) & 1, 103, abort_flag)) break;

            // Q as the B operand (col-major K x N = dims x queries == Q rows [query][dim])
            uint32_t qb[DT][2];
            {
                const uint32_t qbase = sbase + L.q_off + (uint32_t)(qs * kQTile) * pitch + head_off;
#pragma unroll
                for (int kk = 0; kk < DT; ++kk) {
                    if (16 * kk + 16 <= p.D) {
                        const uint32_t a = qbase + (uint32_t)(lane & 7) * pitch + (uint32_t)(16 * kk + 8 * ((lane >> 3) & 1)) * 2u;
                        ldsm_x2(a, qb[kk][0], qb[kk][1]);
                    } else {
                        const uint32_t a = qbase + (uint32_t)(lane & 7) * pitch + (uint32_t)(16 * kk) * 2u;
                        ldsm_x1(a, qb[kk][0]);
                        qb[kk][1] = 0u;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(qempty_bar(qs));

            float m_run[2] = {kNegInf, kNegInf};
            float l_part[2] = {0.f, 0.f};
            float acc[DT][4];
#pragma unroll
            for (int t = 0; t < DT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

            bool ok = true;
            for (int st = 0; st < p.n_stages; ++st, ++stage) {
                const int slot = stage % kStages;
                if (!mbar_wait(full_bar(slot), (stage / kStages) & 1, 104, abort_flag)) { ok = false; break; }
                const uint32_t kbase = sbase + (uint32_t)slot * L.stage_bytes + head_off;
                const uint32_t vbase = kbase + (uint32_t)kKeysPerStage * pitch;

                // S^T = K Q^T : 16 keys x 8 queries
                float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < DT; ++kk) {
                    if (16 * kk + 16 <= p.D) {
                        const uint32_t a = kbase + (uint32_t)((lane & 7) + 8 * ((lane >> 3) & 1)) * pitch +
                                           (uint32_t)(16 * kk + 8 * (lane >> 4)) * 2u;
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4(a, a0, a1, a2, a3);
                        mma16816(c, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
                    } else {
                        const uint32_t a = kbase + (uint32_t)((lane & 7) + 8 * ((lane >> 3) & 1)) * pitch +
                                           (uint32_t)(16 * kk) * 2u;
                        uint32_t a0, a1;
                        ldsm_x2(a, a0, a1);
                        mma1688(c, a0, a1, qb[kk][0]);
                    }
                }
                // scores in log2 units with the causal and queue-length masks
                const int kf0 = st * kKeysPerStage + krow;
                const int kf1 = kf0 + 8;
                float sc[4];
                sc[0] = (kf0 < nk && kf0 <= p.Pk + q0) ? c[0] * p.scale_log2 : kNegInf;
                sc[1] = (kf0 < nk && kf0 <= p.Pk + q0 + 1) ? c[1] * p.scale_log2 : kNegInf;
                sc[2] = (kf1 < nk && kf1 <= p.Pk + q0) ? c[2] * p.scale_log2 : kNegInf;
                sc[3] = (kf1 < nk && kf1 <= p.Pk + q0 + 1) ? c[3] * p.scale_log2 : kNegInf;
                float mx0 = fmaxf(sc[0], sc[2]);
                float mx1 = fmaxf(sc[1], sc[3]);
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                }
                const float mn0 = fmaxf(m_run[0], mx0);
                const float mn1 = fmaxf(m_run[1], mx1);
                // key 0 is visible to every query, so after the first stage mn is finite
                const float al0 = ex2(m_run[0] - mn0);
                const float al1 = ex2(m_run[1] - mn1);
                m_run[0] = mn0;
                m_run[1] = mn1;
                const float p0 = ex2(sc[0] - mn0), p1 = ex2(sc[1] - mn1);
                const float p2 = ex2(sc[2] - mn0), p3 = ex2(sc[3] - mn1);
                // P^T (keys x queries) rounded to bf16; the normaliser sums the rounded values
                const uint32_t x0 = pack_bf16x2(p0, p1);
                const uint32_t x1 = pack_bf16x2(p2, p3);
                l_part[0] = l_part[0] * al0 + (bf16_lo(x0) + bf16_lo(x1));
                l_part[1] = l_part[1] * al1 + (bf16_hi(x0) + bf16_hi(x1));
#pragma unroll
                for (int t = 0; t < DT; ++t) {
                    acc[t][0] *= al0;
                    acc[t][1] *= al1;
                    acc[t][2] *= al0;
                    acc[t][3] *= al1;
                }
                // P^T -> B operand fragments
                const uint32_t pb0 = movm_t(x0);
                const uint32_t pb1 = movm_t(x1);
                // O^T += V^T P^T, 16 head dims per m-tile
#pragma unroll
                for (int t = 0; t < DT; ++t) {
                    if (16 * t + 16 <= p.D) {
                        const int j = lane >> 3;
                        const uint32_t a = vbase + (uint32_t)((lane & 7) + 8 * (j >> 1)) * pitch +
                                           (uint32_t)(16 * t + 8 * (j & 1)) * 2u;
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4_t(a, a0, a1, a2, a3);
                        mma16816(acc[t], a0, a1, a2, a3, pb0, pb1);
                    } else {
                        const uint32_t a = vbase + (uint32_t)((lane & 7) + 8 * ((lane >> 3) & 1)) * pitch +
                                           (uint32_t)(16 * t) * 2u;
                        uint32_t a0, a2;
                        ldsm_x2_t(a, a0, a2);
                        mma16816(acc[t], a0, 0u, a2, 0u, pb0, pb1);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(slot));
            }
            if (!ok) break;

            // normalise and write this head's 8 x D block
            float l0 = l_part[0], l1 = l_part[1];
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l0 += __shfl_xor_sync(0xffffffffu, l0, off);
                l1 += __shfl_xor_sync(0xffffffffu, l1, off);
            }
            const float i0 = 1.f / l0, i1 = 1.f / l1;
            // O^T fragments -> O rows with movmatrix; each lane stores two 4-byte pieces of
            // its query row straight to the output (rows of different frames are a
            // frame-plane apart, so there is nothing to gain from staging them)
            const int qrow = lane >> 2;
            __nv_bfloat16 *orow = p.out + (((long long)b * p.n + qrow) * p.HW + s) * HD +
                                  (long long)(hg * G + w) * p.D + 2 * (lane & 3);
#pragma unroll
            for (int t = 0; t < DT; ++t) {
                // movmatrix is warp-collective: every lane transposes, then stores if its
                // query row exists
                const uint32_t y0 = movm_t(pack_bf16x2(acc[t][0] * i0, acc[t][1] * i1));
                if (qrow < p.n) *reinterpret_cast<uint32_t *>(orow + 16 * t) = y0;
                if (16 * t + 16 <= p.D) {
                    const uint32_t y1 = movm_t(pack_bf16x2(acc[t][2] * i0, acc[t][3] * i1));
                    if (qrow < p.n) *reinterpret_cast<uint32_t *>(orow + 16 * t + 8) = y1;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
uint32_t temporal_pitch(int G, int D)
{
    uint32_t units = (uint32_t)(G * D * 2) / 16u;
    if ((units & 1u) == 0) units += 1;   // odd number of 16-byte units: conflict-free ldmatrix
    return units * 16u;
}

uint32_t temporal_smem_bytes(int G, int D) { return make_layout(temporal_pitch(G, D)).total; }

template <int DT>
static cudaError_t launch_dt(const TemporalParams &p, int grid, cudaStream_t stream)
{
    const uint32_t smem = make_layout(p.pitch).total;
    static int configured_for = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_for != dev) {
        cudaError_t e = cudaFuncSetAttribute(k_temporal_causal<DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)make_layout(temporal_pitch(kMaxTemporalGroup, 16 * DT)).total);
        if (e != cudaSuccess) return e;
        configured_for = dev;
    }
    k_temporal_causal<DT><<<grid, 32 * (p.G + 1), smem, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_temporal(const TemporalParams &p, int grid, cudaStream_t stream)
{
    switch ((p.D + 15) / 16) {
    case 1: return launch_dt<1>(p, grid, stream);
    case 2: return launch_dt<2>(p, grid, stream);
    case 3: return launch_dt<3>(p, grid, stream);
    case 4: return launch_dt<4>(p, grid, stream);
    case 5: return launch_dt<5>(p, grid, stream);
    case 6: return launch_dt<6>(p, grid, stream);
    case 7: return launch_dt<7>(p, grid, stream);
    case 8: return launch_dt<8>(p, grid, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ca2
