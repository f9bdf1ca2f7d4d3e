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
//                Tensor maps view a [frames][HW][H][D] tensor as 4-D (D, H, HW, frames).
//                An operand tile is one 64-column box per full 64 head-dims (128-byte
//                rows, 128-byte swizzle) plus 16-column boxes for the rest (32-byte rows,
//                32-byte swizzle); a head dim that is not a multiple of 16 (72) is
//                zero-padded by the TMA unit itself (columns past D read as zero, so
//                D = 72 runs at K = 80) and rows past HW read as zero.
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

// 32 lanes x 128 consecutive 32-bit columns (two x64 loads, one wait), waited for inside
// the same statement so the compiler cannot read the registers early.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%128];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%129];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]),
          "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]),
          "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]),
          "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]),
          "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]),
          "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]),
          "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]),
          "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]),
          "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
        : "r"(taddr), "r"(taddr + 64u)
        : "memory");
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

// One operand tile (128 rows x padded D) is NA boxes of 64 columns with 128-byte rows and
// the 128-byte swizzle (16 KB each), then NR boxes of 16 columns with 32-byte rows and the
// 32-byte swizzle (4 KB each): NA = NKD / 4, NR = NKD % 4 for NKD = ceil(D / 16).  Wide
// rows keep the TMA unit's row rate off the critical path.
__host__ __device__ constexpr uint32_t tile_bytes(int nkd) { return (nkd / 4) * 16384u + (nkd % 4) * 4096u; }

struct SmemLayout {
    uint32_t q, k0, v0, p, bars, total;
};

__host__ __device__ constexpr SmemLayout spatial_layout(int nkd)
{
    SmemLayout L{};
    L.q = 0;
    L.k0 = L.q + ((tile_bytes(nkd) + 1023u) & ~1023u);
    L.v0 = L.k0 + 2 * ((tile_bytes(nkd) + 1023u) & ~1023u);
    L.p = L.v0 + 2 * ((tile_bytes(nkd) + 1023u) & ~1023u);
    L.bars = L.p + 2 * kRows * kKeys * 2;      // two P buffers
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
    B_PFULL = 11,     // 2: P buffer written (4 softmax warps)
    B_ODONE = 13,     // 2: P V product of a block with this parity done
    B_VREADY = 15,    // 2: V stage landed and its padding column prepared
    B_OSTAGED = 17,   // the 4 softmax warps have written their output rows
    B_COUNT = 18
};

}  // namespace

template <int NKD>
__global__ void __launch_bounds__(kThreads, 1) k_spatial_prefix(const __grid_constant__ SpatialMaps tm,
                                                                  const SpatialParams p)
{
    extern __shared__ uint8_t smem_raw[];
    constexpr SmemLayout L = spatial_layout(NKD);
    constexpr int DP = NKD * 16;                 // padded head dim (MMA N of P V)
    constexpr int NA = NKD / 4;                  // 64-column boxes (128-byte swizzle)
    constexpr int NR = NKD % 4;                  // 16-column boxes (32-byte swizzle)
    constexpr uint32_t TB = (tile_bytes(NKD) + 1023u) & ~1023u;   // bytes per operand tile
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
            mbar_init(bar(B_PFULL + i), 4);
            mbar_init(bar(B_ODONE + i), 1);
            mbar_init(bar(B_VREADY + i), 1);
        }
        mbar_init(bar(B_OSTAGED), 4);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < 2; ++i) {
            prefetch_tmap(&tm.q[i]);
            prefetch_tmap(&tm.k[i]);
            prefetch_tmap(&tm.v[i]);
            prefetch_tmap(&tm.sk[i]);
            prefetch_tmap(&tm.sv[i]);
        }
        prefetch_tmap(&tm.o);
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
    // When D is not a multiple of 16 the P V product has padding columns D..DP-1; column D
    // of every V tile is set to 1.0 so that the tensor core also accumulates the row sum
    // of the (bf16) probabilities into O[:, D], rescaled together with O.
    const bool ones_col = (p.D & 15) != 0;

    if (warp == 0) {
        // ------------------------------- TMA producer ---------------------------------
        // one operand tile: NA wide boxes then NR narrow boxes
        auto load_tile = [&](uint32_t dst, const CUtensorMap *wide, const CUtensorMap *narrow, int row0, int fr,
                             uint32_t bar_addr) {
            for (int a = 0; a < NA; ++a) tma_load_4d(dst + a * 16384u, wide, 64 * a, h, row0, fr, bar_addr);
            for (int r = 0; r < NR; ++r)
                tma_load_4d(dst + NA * 16384u + r * 4096u, narrow, 64 * NA + 16 * r, h, row0, fr, bar_addr);
        };
        auto issue = [&](int j) {
            const int s = j & 1;
            const int src = j / p.nkb;
            const int kb = j - src * p.nkb;
            const CUtensorMap *mk = src == 0 ? tm.k : tm.sk;
            const CUtensorMap *mv = src == 0 ? tm.v : tm.sv;
            const int fr = src == 0 ? b * p.n + f : (src - 1) * p.B + b;
            mbar_expect_tx(bar(B_KFULL + s), tile_bytes(NKD));
            load_tile(sb + L.k0 + s * TB, &mk[0], &mk[1], kb * kKeys, fr, bar(B_KFULL + s));
            mbar_expect_tx(bar(B_VFULL + s), tile_bytes(NKD));
            load_tile(sb + L.v0 + s * TB, &mv[0], &mv[1], kb * kKeys, fr, bar(B_VFULL + s));
        };
        int issued = -1;
        if (lane == 0) {
            mbar_expect_tx(bar(B_QFULL), tile_bytes(NKD));
            load_tile(sb + L.q, &tm.q[0], &tm.q[1], qt * kRows, b * p.n + f, bar(B_QFULL));
            for (int j = 0; j < 2 && j < NB; ++j) issue(j);
        }
        issued = NB < 2 ? NB - 1 : 1;
        __syncwarp();
        for (int j = 0; j < NB; ++j) {
            const int s = j & 1;
            if (!warp_wait(bar(B_VFULL + s), (j >> 1) & 1, 200, abort_flag)) break;
            if (ones_col) {
                // column D of this V tile := 1.0 (bf16 0x3F80), at its swizzled address
                const uint32_t vt = sb + L.v0 + s * TB;
                const int D = p.D;
                for (int r = lane; r < kKeys; r += 32) {
                    uint32_t a;
                    if (D < 64 * NA) {          // inside a 64-column box: 128-byte rows, 128-byte swizzle
                        const int c = (D & 63) >> 3;
                        a = vt + (uint32_t)(D >> 6) * 16384u + (uint32_t)r * 128u +
                            (uint32_t)(((c ^ (r & 7)) << 4) + (D & 7) * 2);
                    } else {                    // inside a 16-column box: 32-byte rows, 32-byte swizzle
                        const int e = D - 64 * NA;
                        a = vt + (uint32_t)NA * 16384u + (uint32_t)(e >> 4) * 4096u + (uint32_t)r * 32u +
                            (uint32_t)(((((e & 15) >> 3) ^ ((r >> 2) & 1)) << 4) + (e & 7) * 2);
                    }
                    asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"((unsigned short)0x3F80) : "memory");
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            int go = 1;
            if (lane == 0) {
                mbar_arrive(bar(B_VREADY + s));
                if (j + 2 < NB) {
                    go = mbar_wait(bar(B_KVEMPTY + s), (j >> 1) & 1, 201, abort_flag) ? 1 : 0;
                    if (go) {
                        issue(j + 2);
                        issued = j + 2;
                    }
                }
            }
            if (!__shfl_sync(0xffffffffu, go, 0)) break;
        }
        // wind-down after an abort: let every issued load land before the CTA exits
        if (lane == 0 && *abort_flag) {
            mbar_wait(bar(B_QFULL), 0, 0, nullptr, 2000000ull);
            for (int j = issued > 1 ? issued - 1 : 0; j <= issued; ++j) {
                mbar_wait(bar(B_KFULL + (j & 1)), (j >> 1) & 1, 0, nullptr, 2000000ull);
                mbar_wait(bar(B_VFULL + (j & 1)), (j >> 1) & 1, 0, nullptr, 2000000ull);
            }
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer -----------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(kRows, kKeys, false, false);
            constexpr uint32_t idesc_pv_w = idesc_bf16(kRows, NA > 0 ? 64 * NA : 16, false, true);
            constexpr uint32_t idesc_pv_n = idesc_bf16(kRows, NR > 0 ? 16 * NR : 16, false, true);
            // K-major operand descriptor of k-step kk inside a tile at `t`
            auto kdesc = [&](uint32_t t, int kk) -> uint64_t {
                if (kk < 4 * NA) return sdesc(t + (kk >> 2) * 16384u + (kk & 3) * 32u, 16, 1024, kSw128);
                return sdesc(t + NA * 16384u + (kk - 4 * NA) * 4096u, 16, 256, kSw32);
            };
            bool ok = mbar_wait(bar(B_QFULL), 0, 211, abort_flag);
            int committed = 0;   // P V products committed
            for (int j = 0; ok && j <= NB; ++j) {
                if (j < NB) {
                    const int s = j & 1;
                    if (!mbar_wait(bar(B_KFULL + s), (j >> 1) & 1, 212, abort_flag)) break;
                    if (j >= 2 && !mbar_wait(bar(B_SFREE + s), ((j - 2) >> 1) & 1, 213, abort_flag)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < NKD; ++kk)
                        tc_mma(tmem + s * kKeys, kdesc(sb + L.q, kk), kdesc(sb + L.k0 + s * TB, kk), idesc_qk,
                               kk > 0 ? 1u : 0u);
                    tc_commit(bar(B_SFULL + s));
                }
                if (j >= 1) {
                    const int jj = j - 1;
                    const int s2 = jj & 1;
                    if (!mbar_wait(bar(B_PFULL + s2), (jj >> 1) & 1, 214, abort_flag)) break;
                    if (!mbar_wait(bar(B_VREADY + s2), (jj >> 1) & 1, 215, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t pbuf = sb + L.p + (uint32_t)s2 * (kRows * kKeys * 2);
                    const uint32_t vt = sb + L.v0 + s2 * TB;
#pragma unroll
                    for (int kk = 0; kk < kKeys / 16; ++kk) {
                        const uint64_t ad = sdesc(pbuf + (kk >> 2) * (kRows * 128) + (kk & 3) * 32, 16, 1024, kSw128);
                        const uint32_t acc = (jj > 0 || kk > 0) ? 1u : 0u;
                        // V is MN-major: 16 keys = 16 rows of each box; wide boxes 64 dims
                        // (128-byte rows, atoms 16 KB apart), narrow boxes 16 dims (32-byte rows)
                        if (NA > 0)
                            tc_mma(tmem_o, ad, sdesc(vt + kk * 2048u, 16384, 1024, kSw128), idesc_pv_w, acc);
                        if (NR > 0)
                            tc_mma(tmem_o + 64 * NA, ad, sdesc(vt + NA * 16384u + kk * 512u, 4096, 256, kSw32),
                                   idesc_pv_n, acc);
                    }
                    tc_commit(bar(B_KVEMPTY + s2));
                    tc_commit(bar(B_ODONE + s2));
                    ++committed;
                }
            }
            // wind-down: the tensor core must be idle before TMEM is released
            if (committed > 0) {
                const int jl = committed - 1;
                mbar_wait(bar(B_ODONE + (jl & 1)), (jl >> 1) & 1, 0, nullptr, 2000000ull);
            }
        }
    } else {
        // ------------------------------- softmax / epilogue ---------------------------
        const int quarter = warp & 3;                     // TMEM lanes 32*quarter ..
        const int row = quarter * 32 + lane;              // query row of this thread
        const uint32_t lane_bits = (uint32_t)(quarter * 32) << 16;
        const float neg_inf = __int_as_float(0xff800000);
        const float scale = p.scale_log2;
        float m_used = neg_inf;     // max (log2 units) the probabilities are taken against
        float l_sum = 0.f;         // row sum, kept here only when there is no padding column
        bool ok = true;
        for (int j = 0; j < NB; ++j) {
            const int s = j & 1;
            const int kb = j % p.nkb;
            const int valid = min(kKeys, p.HW - kb * kKeys);
            if (!warp_wait(bar(B_SFULL + s), (j >> 1) & 1, 221, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[kKeys];
            tmem_ld128(tmem + lane_bits + s * kKeys, sr);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SFREE + s));

            float sv[kKeys];
#pragma unroll
            for (int i = 0; i < kKeys; ++i) sv[i] = __uint_as_float(sr[i]);
            if (valid < kKeys) {
#pragma unroll
                for (int i = 0; i < kKeys; ++i)
                    if (i >= valid) sv[i] = neg_inf;
            }
            float m8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) m8[i] = sv[i];
#pragma unroll
            for (int i = 8; i < kKeys; ++i) m8[i & 7] = fmaxf(m8[i & 7], sv[i]);
            const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * scale;
            float alpha = 1.f;
            const bool upd = mx > m_used + kLazyRescale;
            if (upd) {
                alpha = ex2(m_used - mx);
                m_used = mx;
            }
            // P buffer s was last read by the P V product of block j-2; O may be rescaled
            // only once the product of block j-1 is done
            const bool rescale = j > 0 && __any_sync(0xffffffffu, upd);
            if (rescale) {
                if (!warp_wait(bar(B_ODONE + ((j - 1) & 1)), ((j - 1) >> 1) & 1, 222, abort_flag)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < NKD; ++c) {
                    float o[16];
                    tmem_ld16(tmem_o + lane_bits + 16 * c, o);
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] *= alpha;
                    tmem_st16(tmem_o + lane_bits + 16 * c, o);
                }
                tmem_st_wait();
            } else if (j >= 2) {
                if (!warp_wait(bar(B_ODONE + s), ((j - 2) >> 1) & 1, 223, abort_flag)) { ok = false; break; }
            }
            l_sum *= alpha;
            // probabilities -> bf16 A operand: row-major 128 x 128, two 64-key column groups,
            // 128-byte rows with the 128-byte swizzle (16-byte chunk index ^= row % 8)
            const float neg_m = -m_used;
            const uint32_t prow = sb + L.p + (uint32_t)s * (kRows * kKeys * 2) + (uint32_t)row * 128u;
            float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
            for (int c = 0; c < kKeys / 8; ++c) {
                float e[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) e[i] = ex2(fmaf(sv[8 * c + i], scale, neg_m));
                const uint32_t w0 = pack_bf16x2(e[0], e[1]);
                const uint32_t w1 = pack_bf16x2(e[2], e[3]);
                const uint32_t w2 = pack_bf16x2(e[4], e[5]);
                const uint32_t w3 = pack_bf16x2(e[6], e[7]);
                if (!ones_col) {
                    ls0 += (bf16_lo(w0) + bf16_hi(w0)) + (bf16_lo(w1) + bf16_hi(w1));
                    ls1 += (bf16_lo(w2) + bf16_hi(w2)) + (bf16_lo(w3) + bf16_hi(w3));
                }
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
            if (lane == 0) mbar_arrive(bar(B_PFULL + s));
        }
        // ---- epilogue: O / l -> bf16 -> shared (dense [128][D]) -> one TMA store -------
        if (ok && warp_wait(bar(B_ODONE + ((NB - 1) & 1)), ((NB - 1) >> 1) & 1, 224, abort_flag)) {
            tc_fence_after();
            float o_all[DP];
#pragma unroll
            for (int c = 0; c < NKD; ++c) {
                float o[16];
                tmem_ld16(tmem_o + lane_bits + 16 * c, o);
#pragma unroll
                for (int i = 0; i < 16; ++i) o_all[16 * c + i] = o[i];
            }
            float l = l_sum;
            if (ones_col) {
#pragma unroll
                for (int i = 0; i < DP; ++i)
                    if (i == p.D) l = o_all[i];
            }
            const float inv = 1.f / l;
            uint8_t *orow = sgen + L.q + (size_t)row * (size_t)(p.D * 2);
#pragma unroll
            for (int c = 0; c < DP / 8; ++c) {
                if (8 * c < p.D) {
                    uint4 w;
                    w.x = pack_bf16x2(o_all[8 * c + 0] * inv, o_all[8 * c + 1] * inv);
                    w.y = pack_bf16x2(o_all[8 * c + 2] * inv, o_all[8 * c + 3] * inv);
                    w.z = pack_bf16x2(o_all[8 * c + 4] * inv, o_all[8 * c + 5] * inv);
                    w.w = pack_bf16x2(o_all[8 * c + 6] * inv, o_all[8 * c + 7] * inv);
                    *reinterpret_cast<uint4 *>(orow + 16 * c) = w;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_OSTAGED));
        }
        if (warp == 2 && lane == 0 && mbar_wait(bar(B_OSTAGED), 0, 225, abort_flag)) {
            tma_store_4d(&tm.o, sb + L.q, 0, h, qt * kRows, b * p.n + f);
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
    k_spatial_prefix<NKD><<<grid, kThreads, smem, stream>>>(m, p);
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
