// k_spatial.cu -- prefix-enhanced spatial attention on the 5th-generation tensor cores.
//
// Ca2-VDM ("Ca2-VDM" papernotes page, 关键设计 3): every frame's HW spatial queries attend
// to the frame's own K/V concatenated along the spatial axis with the K/V of the last P'
// clean prefix frames (the spatial cache), an attention map of (HW) x ((P'+1) HW).  Clean
// prefix frames are aligned by self-repeating their own K/V, which leaves softmax
// attention unchanged, so that mode reads the own frame once (n_src = 1).
//
// One CTA computes one 128-query tile of one (video, frame, head):
//   warp 0       TMA producer: Q once, then K and V in 128-key blocks, two stages deep.
//                Tensor maps view a [frames][HW][H][D] tensor as 4-D (D, H, HW, frames);
//                a box is 16 head-dims x 128 tokens with 32-byte swizzle, so a head dim
//                that is not a multiple of 16 (72) is zero-padded by the TMA unit itself
//                (columns past D read as zero) and rows past HW read as zero.
//   warp 1       MMA issuer (one thread) and TMEM owner.  S = Q K^T (M=128, N=128 keys,
//                K = padded D) into one of two TMEM score buffers; O += P V (M=128,
//                N = padded D, K = 128 keys) into a TMEM accumulator.  tcgen05.commit
//                arrives on mbarriers that release the score buffer, the K/V stage and P.
//   warps 2..5   softmax, one thread per query row (TMEM lane): scores come in with
//                tcgen05.ld, the running max is only moved when it grows by more than
//                2^8 (the output is then rescaled in TMEM), probabilities are written to
//                shared memory as the bf16 A operand of the next P V product (128-byte
//                swizzle), and the epilogue normalises O and stores it with one TMA store.
//
// Every mbarrier wait is bounded; a timeout is recorded in the library status word and
// all roles wind down through the common exit, which frees TMEM.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ca2_device.cuh"
#include "ca2_kernels.h"

namespace ca2 {

namespace {

constexpr int kThreads = 192;
constexpr int kRows = 128;           // queries per tile = TMEM lanes
constexpr int kKeys = 128;           // keys per block
constexpr uint32_t kBox = 4096;      // one 16-column x 128-row box, bytes
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSw128 = 2, kSw32 = 6;   // smem-descriptor layout codes
constexpr float kLazyRescale = 8.0f;        // log2 units
// Dynamic shared memory is never below this, so at most one CTA is resident per SM and the
// 512-column TMEM allocation never waits on another CTA.
constexpr uint32_t kMinSmem = 116 * 1024;

// ---- tcgen05 helpers ---------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns, waited for inside the same statement so the
// compiler cannot read the registers early.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32], int base)
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    (void)base;
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor (tcgen05): start, leading/stride byte offsets, layout.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;                 // descriptor version for sm_100
    d |= (uint64_t)layout << 61;
    return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major)
{
    return (1u << 4)                          // D format: f32
           | (1u << 7)                        // A format: bf16
           | (1u << 10)                       // B format: bf16
           | ((a_mn_major ? 1u : 0u) << 15)   // A major-ness
           | ((b_mn_major ? 1u : 0u) << 16)   // B major-ness
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct SmemLayout {
    uint32_t q, k0, v0, p, bars, total;
};

__host__ __device__ constexpr SmemLayout spatial_layout(int nkd)
{
    SmemLayout L{};
    L.q = 0;
    L.k0 = L.q + nkd * kBox;
    L.v0 = L.k0 + 2 * nkd * kBox;
    L.p = ((L.v0 + 2 * nkd * kBox) + 1023u) & ~1023u;
    L.bars = L.p + kRows * kKeys * 2;
    L.total = L.bars + 256 + 1024;   // barriers + slack for the 1024-byte base alignment
    if (L.total < kMinSmem) L.total = kMinSmem;
    return L;
}

// barrier indices
enum : int {
    B_QFULL = 0,
    B_KFULL = 1,      // 2
    B_VFULL = 3,      // 2
    B_KVEMPTY = 5,    // 2
    B_SFULL = 7,      // 2
    B_SFREE = 9,      // 2
    B_PFULL = 11,
    B_ODONE = 12,
    B_OSTAGED = 13,   // the 4 softmax warps have written their output rows
    B_COUNT = 14
};

}  // namespace

template <int NKD>
__global__ void __launch_bounds__(kThreads, 1)
    k_spatial_prefix(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_sk,
                     const __grid_constant__ CUtensorMap tm_sv, const __grid_constant__ CUtensorMap tm_o,
                     const SpatialParams p)
{
    extern __shared__ uint8_t smem_raw[];
    constexpr SmemLayout L = spatial_layout(NKD);
    constexpr int DP = NKD * 16;                 // padded head dim (MMA N of P V)
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;  // 1024-aligned base for the swizzled tiles
    uint8_t *sgen = smem_raw + (sb - raw);
    const uint32_t bars = sb + L.bars;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sgen + L.bars + 8 * B_COUNT);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sgen + L.bars + 8 * B_COUNT + 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // tile -> (b, f, h, qt); query tiles fastest, then frames, so CTAs in flight together
    // share the same spatial-cache K/V in L2
    int t = blockIdx.x;
    const int qt = t % p.q_tiles;
    t /= p.q_tiles;
    const int f = t % p.n;
    t /= p.n;
    const int h = t % p.H;
    const int b = t / p.H;
    const int NB = p.n_src * p.nkb;

    if (threadIdx.x == 0) {
        mbar_init(bar(B_QFULL), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(B_KFULL + i), 1);
            mbar_init(bar(B_VFULL + i), 1);
            mbar_init(bar(B_KVEMPTY + i), 1);
            mbar_init(bar(B_SFULL + i), 1);
            mbar_init(bar(B_SFREE + i), 4);
        }
        mbar_init(bar(B_PFULL), 4);
        mbar_init(bar(B_ODONE), 1);
        mbar_init(bar(B_OSTAGED), 4);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_sk);
        prefetch_tmap(&tm_sv);
        prefetch_tmap(&tm_o);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32((const void *)tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_o = tmem + 2 * kKeys;

    if (warp == 0) {
        // ------------------------------- TMA producer ---------------------------------
        if (lane == 0) {
            int issued = -1;   // last block whose loads were issued
            mbar_expect_tx(bar(B_QFULL), NKD * kBox);
            for (int kk = 0; kk < NKD; ++kk)
                tma_load_4d(sb + L.q + kk * kBox, &tm_q, 16 * kk, h, qt * kRows, b * p.n + f, bar(B_QFULL));
            for (int j = 0; j < NB; ++j) {
                const int s = j & 1;
                if (j >= 2 && !mbar_wait(bar(B_KVEMPTY + s), ((j - 2) >> 1) & 1, 201, abort_flag)) break;
                const int src = j / p.nkb;
                const int kb = j - src * p.nkb;
                const CUtensorMap *mk = src == 0 ? &tm_k : &tm_sk;
                const CUtensorMap *mv = src == 0 ? &tm_v : &tm_sv;
                const int fr = src == 0 ? b * p.n + f : (src - 1) * p.B + b;
                mbar_expect_tx(bar(B_KFULL + s), NKD * kBox);
                for (int kk = 0; kk < NKD; ++kk)
                    tma_load_4d(sb + L.k0 + (s * NKD + kk) * kBox, mk, 16 * kk, h, kb * kKeys, fr, bar(B_KFULL + s));
                mbar_expect_tx(bar(B_VFULL + s), NKD * kBox);
                for (int kk = 0; kk < NKD; ++kk)
                    tma_load_4d(sb + L.v0 + (s * NKD + kk) * kBox, mv, 16 * kk, h, kb * kKeys, fr, bar(B_VFULL + s));
                issued = j;
            }
            // wind-down after an abort: let every issued load land before the CTA exits
            if (*abort_flag) {
                mbar_wait(bar(B_QFULL), 0, 0, nullptr, 2000000ull);
                for (int j = issued > 1 ? issued - 1 : 0; j <= issued; ++j) {
                    mbar_wait(bar(B_KFULL + (j & 1)), (j >> 1) & 1, 0, nullptr, 2000000ull);
                    mbar_wait(bar(B_VFULL + (j & 1)), (j >> 1) & 1, 0, nullptr, 2000000ull);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer -----------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(kRows, kKeys, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16(kRows, DP, false, true);
            bool ok = mbar_wait(bar(B_QFULL), 0, 211, abort_flag);
            int committed = 0;   // P V products committed
            for (int j = 0; ok && j <= NB; ++j) {
                if (j < NB) {
                    const int s = j & 1;
                    if (!mbar_wait(bar(B_KFULL + s), (j >> 1) & 1, 212, abort_flag)) break;
                    if (j >= 2 && !mbar_wait(bar(B_SFREE + s), ((j - 2) >> 1) & 1, 213, abort_flag)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < NKD; ++kk) {
                        const uint64_t ad = sdesc(sb + L.q + kk * kBox, 16, 256, kSw32);
                        const uint64_t bd = sdesc(sb + L.k0 + (s * NKD + kk) * kBox, 16, 256, kSw32);
                        tc_mma(tmem + s * kKeys, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(bar(B_SFULL + s));
                }
                if (j >= 1) {
                    const int jj = j - 1;
                    const int s2 = jj & 1;
                    if (!mbar_wait(bar(B_PFULL), jj & 1, 214, abort_flag)) break;
                    if (!mbar_wait(bar(B_VFULL + s2), (jj >> 1) & 1, 215, abort_flag)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kKeys / 16; ++kk) {
                        const uint64_t ad = sdesc(sb + L.p + (kk >> 2) * (kRows * 128) + (kk & 3) * 32, 16, 1024, kSw128);
                        const uint64_t bd = sdesc(sb + L.v0 + s2 * NKD * kBox + kk * 512, kBox, 256, kSw32);
                        tc_mma(tmem_o, ad, bd, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(bar(B_KVEMPTY + s2));
                    tc_commit(bar(B_ODONE));
                    ++committed;
                }
            }
            // wind-down: the tensor core must be idle before TMEM is released
            if (committed > 0) mbar_wait(bar(B_ODONE), (committed - 1) & 1, 0, nullptr, 2000000ull);
        }
    } else {
        // ------------------------------- softmax / epilogue ---------------------------
        const int quarter = warp & 3;                     // TMEM lanes 32*quarter ..
        const int row = quarter * 32 + lane;              // query row of this thread
        const uint32_t lane_bits = (uint32_t)(quarter * 32) << 16;
        const float neg_inf = __int_as_float(0xff800000);
        float m_used = neg_inf;
        float l_sum = 0.f;
        bool ok = true;
        for (int j = 0; j < NB; ++j) {
            const int s = j & 1;
            const int kb = j % p.nkb;
            const int valid = min(kKeys, p.HW - kb * kKeys);
            if (!mbar_wait(bar(B_SFULL + s), (j >> 1) & 1, 221, abort_flag)) { ok = false; break; }
            tc_fence_after();
            float sv[kKeys];
#pragma unroll
            for (int c = 0; c < kKeys / 32; ++c) {
                float tmp[32];
                tmem_ld32(tmem + lane_bits + s * kKeys + 32 * c, tmp, 0);
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[32 * c + i] = tmp[i];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SFREE + s));

            float mx = neg_inf;
#pragma unroll
            for (int i = 0; i < kKeys; ++i) {
                const float x = (i < valid) ? sv[i] * p.scale_log2 : neg_inf;
                sv[i] = x;
                mx = fmaxf(mx, x);
            }
            float alpha = 1.f;
            const bool upd = mx > m_used + kLazyRescale;
            if (upd) {
                alpha = ex2(m_used - mx);
                m_used = mx;
            }
            if (j > 0) {
                // the previous P V product must be done before O or P are touched
                if (!mbar_wait(bar(B_ODONE), (j - 1) & 1, 222, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, upd)) {
#pragma unroll
                    for (int c = 0; c < NKD; ++c) {
                        float o[16];
                        tmem_ld16(tmem_o + lane_bits + 16 * c, o);
#pragma unroll
                        for (int i = 0; i < 16; ++i) o[i] *= alpha;
                        tmem_st16(tmem_o + lane_bits + 16 * c, o);
                    }
                    tmem_st_wait();
                }
            }
            l_sum *= alpha;
            // probabilities -> bf16 A operand: row-major 128 x 128, two 64-key column groups,
            // 128-byte rows with the 128-byte swizzle (16-byte chunk index ^= row % 8)
            // The normaliser sums the same bf16-rounded probabilities the P V product uses,
            // so the weights applied to V form an exact distribution.
            const uint32_t prow = sb + L.p + (uint32_t)row * 128u;
            float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
            for (int c = 0; c < kKeys / 8; ++c) {
                float e[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) e[i] = ex2(sv[8 * c + i] - m_used);
                const uint32_t w0 = pack_bf16x2(e[0], e[1]);
                const uint32_t w1 = pack_bf16x2(e[2], e[3]);
                const uint32_t w2 = pack_bf16x2(e[4], e[5]);
                const uint32_t w3 = pack_bf16x2(e[6], e[7]);
                ls0 += (bf16_lo(w0) + bf16_hi(w0)) + (bf16_lo(w1) + bf16_hi(w1));
                ls1 += (bf16_lo(w2) + bf16_hi(w2)) + (bf16_lo(w3) + bf16_hi(w3));
                const uint32_t addr = prow + (uint32_t)(c >> 3) * (kRows * 128u) +
                                      (uint32_t)(((c & 7) ^ (row & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(w0), "r"(w1), "r"(w2),
                             "r"(w3)
                             : "memory");
            }
            l_sum += ls0 + ls1;
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_PFULL));
        }
        // ---- epilogue: O / l -> bf16 -> shared (dense [128][D]) -> one TMA store -------
        if (ok && mbar_wait(bar(B_ODONE), (NB - 1) & 1, 223, abort_flag)) {
            tc_fence_after();
            const float inv = 1.f / l_sum;
            uint8_t *orow = sgen + L.q + (size_t)row * (size_t)(p.D * 2);
#pragma unroll
            for (int c = 0; c < NKD; ++c) {
                float o[16];
                tmem_ld16(tmem_o + lane_bits + 16 * c, o);
                if (16 * c < p.D) {
                    uint4 w;
                    w.x = pack_bf16x2(o[0] * inv, o[1] * inv);
                    w.y = pack_bf16x2(o[2] * inv, o[3] * inv);
                    w.z = pack_bf16x2(o[4] * inv, o[5] * inv);
                    w.w = pack_bf16x2(o[6] * inv, o[7] * inv);
                    *reinterpret_cast<uint4 *>(orow + 32 * c) = w;
                }
                if (16 * c + 8 < p.D) {
                    uint4 w;
                    w.x = pack_bf16x2(o[8] * inv, o[9] * inv);
                    w.y = pack_bf16x2(o[10] * inv, o[11] * inv);
                    w.z = pack_bf16x2(o[12] * inv, o[13] * inv);
                    w.w = pack_bf16x2(o[14] * inv, o[15] * inv);
                    *reinterpret_cast<uint4 *>(orow + 32 * c + 16) = w;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_OSTAGED));
        }
        if (warp == 2 && lane == 0 && mbar_wait(bar(B_OSTAGED), 0, 224, abort_flag)) {
            tma_store_4d(&tm_o, sb + L.q, 0, h, qt * kRows, b * p.n + f);
            bulk_commit();
            bulk_wait<0>();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

uint32_t spatial_smem_bytes(int D)
{
    const int nkd = (D + 15) / 16;
    return spatial_layout(nkd).total;
}

template <int NKD>
static cudaError_t launch_nkd(const SpatialMaps &m, const SpatialParams &p, cudaStream_t stream)
{
    constexpr uint32_t smem = spatial_layout(NKD).total;
    static int configured_for = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_for != dev) {
        cudaError_t e =
            cudaFuncSetAttribute(k_spatial_prefix<NKD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured_for = dev;
    }
    const unsigned grid = (unsigned)(p.B * p.n * p.H * p.q_tiles);
    k_spatial_prefix<NKD><<<grid, kThreads, smem, stream>>>(m.q, m.k, m.v, m.sk, m.sv, m.o, p);
    return cudaGetLastError();
}

cudaError_t launch_spatial(const SpatialMaps &m, const SpatialParams &p, cudaStream_t stream)
{
    switch ((p.D + 15) / 16) {
    case 1: return launch_nkd<1>(m, p, stream);
    case 2: return launch_nkd<2>(m, p, stream);
    case 3: return launch_nkd<3>(m, p, stream);
    case 4: return launch_nkd<4>(m, p, stream);
    case 5: return launch_nkd<5>(m, p, stream);
    case 6: return launch_nkd<6>(m, p, stream);
    case 7: return launch_nkd<7>(m, p, stream);
    case 8: return launch_nkd<8>(m, p, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ca2
