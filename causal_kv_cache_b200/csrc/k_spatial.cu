// k_spatial.cu -- prefix-enhanced spatial attention on the 5th-generation tensor cores.
//
// Ca2-VDM ("Ca2-VDM" papernotes page, 关键设计 3): every frame's HW spatial queries attend
// to the frame's own K/V concatenated along the spatial axis with the K/V of the last P'
// clean prefix frames (the spatial cache), an attention map of (HW) x ((P'+1) HW).  Clean
// prefix frames are aligned by self-repeating their own K/V, which leaves softmax
// attention unchanged, so that mode reads the own frame once (n_src = 1).
//
// One CTA computes two 128-query tiles (A and B) of one (video, frame, head); each K/V
// block is loaded once and used by both tiles.  Twelve warps:
//   warp 0       TMA producer: both Q tiles, then K and V blocks of 128 keys into two
//                independent rings (K is released as soon as both QK^T products have read
//                it, V after both P V products).  An operand tile is ceil(D/32) boxes of 32
//                head-dims x 128 tokens (64-byte rows, 64-byte swizzle); columns past D
//                (72 -> 96) and rows past HW are zero-filled by the TMA unit.  Warp 3
//                converts each landed V tile in place to fp16, and when D is not a multiple
//                of 32 sets padding column D to 1.0, so the P V product also accumulates the
//                row sum of the probabilities into O[:, D].  P V runs in fp16 x fp16: the
//                probabilities carry 11 significant bits, where bf16 P (8 bits) put an error
//                of the order of the output's own bf16 rounding into every output.
//   warps 1, 2   MMA issuers of tile A and tile B (the whole warp runs the loop, one
//                elected lane issues; warp 1 owns the 512 TMEM columns).  A divergent
//                single thread issued about one tcgen05.mma per ~100 cycles, the whole warp
//                with warp-uniform operands reaches the tensor rate.  The
//                tile's next QK^T is issued as soon as its softmax warps have read the
//                current scores, and its P V product chunk by chunk as the probabilities
//                land, so the tensor core works while the exponentials run.
//   warp 3       prepares each landed V tile (fp16 conversion and the padding column, below).
//   warps 4-11   softmax: 4 warps per tile, one thread per query row (its TMEM lane; warp
//                % 4 selects the lane quarter) holding all 128 scores of a block in
//                registers, so the row max needs no exchange.  The exponential unit
//                (measured 16 lanes/clock/SM) is the scarce pipe; both tiles' warps share
//                it, so one warp's stalls are filled by the other's work.  Each tile writes
//                its bf16 probabilities into its own buffer in shared memory (the A operand
//                of the P V product) and hands a whole block to its issuer with one proxy
//                fence, so the tiles never wait for each other; at D = 128 they are written
//                over the tile's scores in TMEM and handed over chunk by chunk.
//                The running max moves only when it grows by more than 2^8 (O is then
//                rescaled in TMEM).
//                Epilogue: O / l -> bf16 rows staged in the tile's spent Q buffer -> one
//                TMA store of 32 rows per warp.
//
// Every mbarrier wait is bounded; a timeout is recorded in the library status word and
// all roles wind down through the common exit, which frees TMEM.
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ca2_device.cuh"
#include "ca2_kernels.h"
#include "ca2_tcgen05.cuh"

namespace ca2 {

namespace {

constexpr int kThreads = 384;        // 12 warps
constexpr int kRows = 128;           // queries per tile = TMEM lanes
constexpr int kKeys = 128;           // keys per block
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSw64 = 4;               // smem-descriptor layout code: 64-byte swizzle
constexpr float kLazyRescale = 8.0f;        // log2 units

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// max(a, b, c) in one instruction (three-input max of sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 32 lanes x 128 consecutive 32-bit columns (two x64 loads, one wait).
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

// One operand tile (128 rows x padded D) is NB32 = ceil(D / 32) boxes of 32 columns with
// 64-byte rows and the 64-byte swizzle (8 KB each).  64-byte rows stream at full speed
// through the TMA unit, and one layout serves both products: K-major for Q and K (a
// 16-column k-step is half a swizzled row) and MN-major for V, so P V is a single MMA of
// N = 32 * NB32 per 16 keys.  Columns past D (72 -> 96) read as zero.
__host__ __device__ constexpr int n32(int nkd) { return (nkd + 1) / 2; }
__host__ __device__ constexpr uint32_t tile_bytes(int nkd) { return n32(nkd) * 8192u; }
__host__ __device__ constexpr uint32_t tile_slot(int nkd) { return (tile_bytes(nkd) + 1023u) & ~1023u; }
// Probabilities in shared memory (one 128 x 128 bf16 buffer per tile, four boxes of 32 keys in
// the same 64-byte-swizzled layout as Q) when the padded head dim is at most 96; at 128 they
// are written over the tile's own scores in TMEM instead (no room for both buffers).
__host__ __device__ constexpr bool p_in_smem(int nkd) { return n32(nkd) <= 3; }
__host__ __device__ constexpr uint32_t p_bytes(int nkd) { return p_in_smem(nkd) ? 2u * 4u * 8192u : 0u; }
// K and V ring depth: three blocks when it fits in shared memory, else two
__host__ __device__ constexpr int kv_stages(int nkd)
{
    return 8u * tile_slot(nkd) + p_bytes(nkd) + 1536u <= 232448u ? 3 : 2;
}

struct SmemLayout {
    uint32_t q0, k0, v0, p0, bars, total;
};

__host__ __device__ constexpr SmemLayout spatial_layout(int nkd)
{
    SmemLayout L{};
    L.q0 = 0;                                            // Q of tile A, then tile B
    L.k0 = 2 * tile_slot(nkd);
    L.v0 = L.k0 + kv_stages(nkd) * tile_slot(nkd);
    L.p0 = L.v0 + kv_stages(nkd) * tile_slot(nkd);     // P of tile A, then tile B (32 KB each)
    L.bars = L.p0 + p_bytes(nkd);
    L.total = L.bars + 512 + 1024;   // barriers and flags; slack for the 1024-byte base alignment
    return L;
}

// TMEM columns (512 allocated).  With the probabilities in shared memory (padded head dim DP
// at most 96) TMEM holds each tile's scores and output only:
//   S_A [0,128)  S_B [128,256)  O_A [256,256+DP)  O_B [256+DP,256+2DP)
// so a tile's next scores can be computed while its probabilities are still being written and
// read.  With DP = 128, P is written over the tile's own scores and the next QK^T waits for
// the P V product.
template <int NB32>
struct TmemMap {
    static constexpr int DP = 32 * NB32;
    static constexpr bool kPSmem = NB32 <= 3;
    __host__ __device__ static constexpr uint32_t s(int X) { return (uint32_t)X * 128u; }
    __host__ __device__ static constexpr uint32_t p(int X) { return (uint32_t)X * 128u; }   // P over S (DP = 128)
    __host__ __device__ static constexpr uint32_t o(int X)
    {
        return kPSmem ? 256u + (uint32_t)(X * DP) : 256u + (uint32_t)X * 128u;
    }
};
static_assert(TmemMap<3>::o(1) + 96 <= kTmemCols, "TMEM map overflows");
static_assert(TmemMap<4>::o(1) + 128 <= kTmemCols, "TMEM map overflows");
static_assert(TmemMap<3>::kPSmem == p_in_smem(5) && !TmemMap<4>::kPSmem, "P placement mismatch");
static_assert(8 * 35 + 16 <= 512, "barrier region overflows");

constexpr int kChunks = 4;            // probability chunks per block: 32 keys = 16 P columns each
constexpr int kSoftmaxWarp0 = 4;      // warps 4..7 tile A, 8..11 tile B

// barrier indices (K/V rings have up to three stages; X = tile, c = probability chunk)
enum : int {
    B_QFULL = 0,      // Q of tile A (tile B's Q has its own barrier, B_QFULLB)
    B_KFULL = 1,      // 3
    B_KEMPTY = 4,     // 3: both tiles' QK^T of the block are done (2 commits)
    B_VFULL = 7,      // 3
    B_VREADY = 10,    // 3: padding column prepared
    B_VEMPTY = 13,    // 3: both tiles' P V of the block are done (2 commits)
    B_SFULL = 16,     // 2 [X]: scores in TMEM
    B_SFREE = 18,     // 2 [X]: every softmax warp of the tile has read the scores (4 warps)
    B_PFULL = 20,     // 8 [X][c]: probabilities written (4 warps): per chunk in TMEM, or the
                      //           whole block in shared memory ([X][0] only)
    B_UNUSED = 28,    // 2 (free)
    B_ODONE = 30,     // 2 [X]: P V of the block done (all prior products of the tile)
    B_FIN = 32,       // 2 [X]: every product the tile's issuer launched is done
    B_QFULLB = 34,    // Q of tile B
    B_COUNT = 35
};
static_assert(8 * B_COUNT + 12 <= 512, "barrier area");

}  // namespace

template <int NKD>
__global__ void __launch_bounds__(kThreads, 1) k_spatial_prefix(const __grid_constant__ SpatialMaps tm,
                                                   const SpatialParams p)
{
    extern __shared__ uint8_t smem_raw[];
    constexpr SmemLayout L = spatial_layout(NKD);
    constexpr int NS = kv_stages(NKD);
    constexpr int NB32 = n32(NKD);               // 32-column boxes per operand tile
    constexpr int DP = 32 * NB32;                // P V width (padded head dim)
    constexpr uint32_t TB = tile_slot(NKD);
    using TM = TmemMap<NB32>;
    constexpr bool kPSmem = TM::kPSmem;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;  // 1024-aligned base for the swizzled tiles
    uint8_t *sgen = smem_raw + (sb - raw);
    const uint32_t bars = sb + L.bars;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sgen + L.bars + 8 * B_COUNT);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sgen + L.bars + 8 * B_COUNT + 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // CTA -> (b, f, h, pair of query tiles); tile pairs fastest, then frames, so CTAs in
    // flight together share the same spatial-cache K/V in L2
    int t = blockIdx.x;
    const int qp = t % p.q_pairs;
    t /= p.q_pairs;
    const int f = t % p.n;
    t /= p.n;
    const int h = t % p.H;
    const int b = t / p.H;
    const int NB = p.n_src * p.nkb;
    const int row0 = qp * 2 * kRows;             // first query row of tile A; tile B follows

    // one operand tile: NB32 boxes of 32 columns
    auto load_tile = [&](uint32_t dst, const CUtensorMap *map, int r0, int fr, uint32_t bar_addr) {
        for (int a = 0; a < NB32; ++a) tma_load_4d(dst + a * 8192u, map, 32 * a, h, r0, fr, bar_addr);
    };
    // key block j -> (tensor map, first key row, frame index).  The spatial-cache frames
    // come first and the own frame last: cache frames are shared by the n frames' CTAs
    // (mostly L2 hits), so the first blocks arrive quickly, and the own frame's blocks,
    // unique to this CTA and read from HBM, stream in while the cache blocks are computed.
    // The order only changes the summation order of the online softmax.
    auto kv_src = [&](int j, const CUtensorMap *&mk, const CUtensorMap *&mv, int &r, int &fr) {
        const int si = j / p.nkb;
        const int src = p.n_src > 1 ? (si + 1) % p.n_src : 0;
        r = (j - si * p.nkb) * kKeys;
        mk = src == 0 ? &tm.k : &tm.sk;
        mv = src == 0 ? &tm.v : &tm.sv;
        fr = src == 0 ? b * p.n + f : (src - 1) * p.B + b;
    };

    if (threadIdx.x == 0) {
        mbar_init(bar(B_QFULL), 1);
        mbar_init(bar(B_QFULLB), 1);
        for (int i = 0; i < NS; ++i) {
            mbar_init(bar(B_KFULL + i), 1);
            mbar_init(bar(B_KEMPTY + i), 2);
            mbar_init(bar(B_VFULL + i), 1);
            mbar_init(bar(B_VREADY + i), 1);
            mbar_init(bar(B_VEMPTY + i), 2);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(B_SFULL + i), 1);
            mbar_init(bar(B_SFREE + i), 4);
            mbar_init(bar(B_ODONE + i), 1);
            mbar_init(bar(B_FIN + i), 1);
        }
        for (int i = 0; i < 2 * kChunks; ++i) mbar_init(bar(B_PFULL + i), 4);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm.q);
        prefetch_tmap(&tm.k);
        prefetch_tmap(&tm.v);
        prefetch_tmap(&tm.sk);
        prefetch_tmap(&tm.sv);
        prefetch_tmap(&tm.o);
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
    if (threadIdx.x == 0) {
        // issue order Q_A, K(0), Q_B, V(0), each on its own barrier: tile A's first QK^T needs
        // only the first two, so it starts while the rest land (measured 24.2 -> 23.2 us per
        // launch against one barrier for both Q tiles ahead of K(0))
        mbar_expect_tx(bar(B_QFULL), tile_bytes(NKD));
        load_tile(sb + L.q0, &tm.q, row0, b * p.n + f, bar(B_QFULL));
        const CUtensorMap *mk = nullptr, *mv = nullptr;
        int r = 0, fr = 0;
        if (NB > 0) {
            kv_src(0, mk, mv, r, fr);
            mbar_expect_tx(bar(B_KFULL), tile_bytes(NKD));
            load_tile(sb + L.k0, mk, r, fr, bar(B_KFULL));
        }
        mbar_expect_tx(bar(B_QFULLB), tile_bytes(NKD));
        load_tile(sb + L.q0 + TB, &tm.q, row0 + kRows, b * p.n + f, bar(B_QFULLB));
        if (NB > 0) {
            mbar_expect_tx(bar(B_VFULL), tile_bytes(NKD));
            load_tile(sb + L.v0, mv, r, fr, bar(B_VFULL));
        }
    }
    const uint32_t tmem = *tmem_slot;
    // When D is not a multiple of 32 the P V product has padding columns D..DP-1; column D
    // of every V tile is set to 1.0 so that the tensor core also accumulates the row sum
    // of the (bf16) probabilities into O[:, D], rescaled together with O.
    const bool ones_col = (p.D & 31) != 0;
    // columns the P V product actually needs: the head dims plus the ones column, rounded up
    // to the MMA's N granule of 16 (80 of the 96 loaded at D = 72); the rest stay unused
    const int dpv = ((p.D + (ones_col ? 1 : 0) + 15) & ~15) < DP ? ((p.D + (ones_col ? 1 : 0) + 15) & ~15) : DP;

    if (warp == 0) {
        // ------------------------------- TMA producer (one warp) ----------------------
        // lane 0 issues the loads (block 0 went out with the barrier setup) as fast as
        // ring slots free up.
        int issued_k = NB > 0 ? 0 : -1, issued_v = issued_k;
        bool ok = true;
        for (int j = 1; ok && j < NB; ++j) {
            const int s = j % NS;
            const int u = j / NS;
            const CUtensorMap *mk, *mv;
            int r, fr;
            kv_src(j, mk, mv, r, fr);
            if (j >= NS && !warp_wait(bar(B_KEMPTY + s), (u - 1) & 1, 201, abort_flag)) { ok = false; break; }
            if (lane == 0) {
                mbar_expect_tx(bar(B_KFULL + s), tile_bytes(NKD));
                load_tile(sb + L.k0 + s * TB, mk, r, fr, bar(B_KFULL + s));
            }
            issued_k = j;
            if (j >= NS && !warp_wait(bar(B_VEMPTY + s), (u - 1) & 1, 202, abort_flag)) { ok = false; break; }
            if (lane == 0) {
                mbar_expect_tx(bar(B_VFULL + s), tile_bytes(NKD));
                load_tile(sb + L.v0 + s * TB, mv, r, fr, bar(B_VFULL + s));
            }
            issued_v = j;
        }
        // wind-down after an abort: let every issued load land before the CTA exits
        // (each ring slot's last use is the most recent phase of its barrier)
        if (lane == 0 && *abort_flag) {
            mbar_wait(bar(B_QFULL), 0, 0, nullptr, 2000000ull);
            mbar_wait(bar(B_QFULLB), 0, 0, nullptr, 2000000ull);
            for (int j = issued_k; j >= 0 && j > issued_k - NS; --j)
                mbar_wait(bar(B_KFULL + j % NS), (j / NS) & 1, 0, nullptr, 2000000ull);
            for (int j = issued_v; j >= 0 && j > issued_v - NS; --j)
                mbar_wait(bar(B_VFULL + j % NS), (j / NS) & 1, 0, nullptr, 2000000ull);
        }
    } else if (warp <= 2) {
        // ------------------------- MMA issuers: warp 1 tile A, warp 2 tile B ------------
        // The whole warp runs the loop with warp-uniform operands; one elected lane issues.
        const int X = warp - 1;
        const uint32_t tm_u = __shfl_sync(0xffffffffu, tmem, 0);
        constexpr uint32_t idesc_qk = idesc_bf16(kRows, kKeys, false, false);
        const uint32_t idesc_pv = idesc_f16(kRows, dpv, false, true);       // P and V both fp16
        // Descriptors are built once; a k-step only adds its byte offset / 16 to the
        // start-address field (addresses stay below 256 KB, so no carry leaves it).
        // K-major (Q, K): 8-row groups 512 B apart; k-step kk = box kk/2, +32 B for odd kk.
        // MN-major (V): atoms of 32 head-dims 8 KB apart (LBO), 8-key groups 512 B apart.
        const uint64_t dq = sdesc(sb + L.q0 + X * TB, 16, 512, kSw64);
        const uint64_t dk0 = sdesc(sb + L.k0, 16, 512, kSw64);
        const uint64_t dv0 = sdesc(sb + L.v0, 8192, 512, kSw64);
        // P_X in shared memory: K-major like Q (keys along the swizzled rows)
        const uint64_t dp = sdesc(sb + L.p0 + (uint32_t)X * 32768u, 16, 512, kSw64);
        auto koff = [](int kk) -> uint64_t { return (uint64_t)(((kk >> 1) * 8192 + (kk & 1) * 32) >> 4); };
        const uint32_t s_x = tm_u + TM::s(X), p_x = tm_u + TM::p(X), o_x = tm_u + TM::o(X);
        // S_X = Q_X K(j)^T; the commits release the scores to the softmax warps and
        // (with the other tile's commit) the K slot to the producer
        auto issue_qk = [&](int j) {
            const uint64_t bk = dk0 + (uint64_t)(((j % NS) * TB) >> 4);
#pragma unroll
            for (int kk = 0; kk < NKD; ++kk)
                tc_mma_ss_w(s_x, dq + koff(kk), bk + koff(kk), idesc_qk, kk > 0 ? 1u : 0u);
            tc_commit_w(bar(B_SFULL + X));
            tc_commit_w(bar(B_KEMPTY + j % NS));
        };
        // O_X (+)= P chunk c V(j), keys 32c..32c+31 = k-steps 2c and 2c+1: from P_X's box c
        // in shared memory, or (P over S) from TMEM columns 16c..16c+15 (two bf16 per column)
        auto issue_pv = [&](int j, int c) {
            const uint64_t bv = dv0 + (uint64_t)(((j % NS) * TB) >> 4);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int kk = 2 * c + e;
                if constexpr (kPSmem)
                    tc_mma_ss_w(o_x, dp + koff(kk), bv + (uint64_t)((kk * 1024) >> 4), idesc_pv,
                                (j > 0 || kk > 0) ? 1u : 0u);
                else
                    tc_mma_ts_w(o_x, p_x + 8 * kk, bv + (uint64_t)((kk * 1024) >> 4), idesc_pv,
                                (j > 0 || kk > 0) ? 1u : 0u);
            }
        };
        bool ok = warp_wait(bar(X ? B_QFULLB : B_QFULL), 0, 211, abort_flag) && warp_wait(bar(B_KFULL), 0, 212, abort_flag);
        if (ok) {
            tc_fence_after();
            issue_qk(0);
        }
        for (int j = 0; ok && j < NB; ++j) {
            if (kPSmem && j + 1 < NB) {
                // the tile's score region is free once its softmax warps have read S(j):
                // compute S(j+1) while they exponentiate
                const int j1 = j + 1;
                if (!warp_wait(bar(B_SFREE + X), j & 1, 213, abort_flag) ||
                    !warp_wait(bar(B_KFULL + j1 % NS), (j1 / NS) & 1, 214, abort_flag))
                    break;
                tc_fence_after();
                issue_qk(j1);
            }
            if (!warp_wait(bar(B_VREADY + j % NS), (j / NS) & 1, 215, abort_flag)) break;
            bool okc = true;
            if constexpr (kPSmem) {
                // the whole block's probabilities at once (one proxy fence per softmax warp)
                okc = warp_wait(bar(B_PFULL + kChunks * X), j & 1, 216, abort_flag);
                if (okc) {
                    tc_fence_after();
                    for (int c = 0; c < kChunks; ++c) issue_pv(j, c);
                }
            } else {
                for (int c = 0; c < kChunks; ++c) {
                    if (!warp_wait(bar(B_PFULL + kChunks * X + c), j & 1, 216, abort_flag)) { okc = false; break; }
                    tc_fence_after();
                    issue_pv(j, c);
                }
            }
            if (!okc) break;
            tc_commit_w(bar(B_ODONE + X));
            tc_commit_w(bar(B_VEMPTY + j % NS));
            if (!kPSmem && j + 1 < NB) {
                // P was written over S: the next scores follow the P V product
                const int j1 = j + 1;
                if (!warp_wait(bar(B_KFULL + j1 % NS), (j1 / NS) & 1, 214, abort_flag)) break;
                tc_fence_after();
                issue_qk(j1);
            }
        }
        // wind-down: the tensor core must be idle before TMEM is released
        tc_commit_w(bar(B_FIN + X));
        mbar_wait(bar(B_FIN + X), 0, 0, nullptr, 2000000ull);
        __syncwarp();
    } else if (warp == 3) {
        // ------------------------------- V preparation (one warp) ---------------------
        // The spatial cache holds V in fp16 already (written so once per AR step); a V tile
        // of the frame's own K/V (bf16, from the caller) is converted in place to fp16 (exact
        // for |v| in [2^-14, 65504]; smaller values become fp16 subnormals, within 2^-25 of
        // v): the 16-byte pieces holding columns < D, four rows per lane, whatever their
        // swizzled position (64-byte rows, 16-byte piece index ^= (row >> 1) & 3).  Values
        // beyond the fp16 range (|v| >= 65536 in bf16, inf, NaN) are recorded in the library
        // status word (ca2_device_status reports CA2_ERR_RANGE).  When D is not a multiple of
        // 32, column D := 1.0 (fp16 0x3C00), so the P V product also accumulates the row sum.
        const int D = p.D;
        const int pieces = D >> 3;                        // 16-byte pieces of a row holding columns < D
        uint32_t vmax = 0;                                // per-half max of |v| bits seen
        auto prep = [&](int jv) -> bool {
            const int s = jv % NS;
            if (!warp_wait(bar(B_VFULL + s), (jv / NS) & 1, 203, abort_flag)) return false;
            const uint32_t vt = sb + L.v0 + s * TB;
            // block jv comes from the own frame when its source index is 0 (see kv_src)
            const bool own = p.n_src == 1 || (jv / p.nkb + 1) % p.n_src == 0;
            // 12 pieces in flight per lane: pieces q0..q0+2 of the lane's four rows
            static_assert(kKeys == 4 * 32, "four rows per lane");
            for (int q0 = 0; own && q0 < pieces; q0 += 3) {
                uint32_t w[3][4][4];
                uint32_t adr[3][4];
#pragma unroll
                for (int dq = 0; dq < 3; ++dq)
#pragma unroll
                    for (int ri = 0; ri < 4; ++ri) {
                        const int q = q0 + dq, r = lane + 32 * ri;
                        adr[dq][ri] = vt + (uint32_t)r * 64u + (uint32_t)(q >> 2) * 8192u +
                                      ((((uint32_t)q & 3u) ^ (uint32_t)((r >> 1) & 3)) << 4);
                        if (q < pieces)
                            asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                                         : "=r"(w[dq][ri][0]), "=r"(w[dq][ri][1]), "=r"(w[dq][ri][2]), "=r"(w[dq][ri][3])
                                         : "r"(adr[dq][ri]));
                    }
#pragma unroll
                for (int dq = 0; dq < 3; ++dq)
#pragma unroll
                    for (int ri = 0; ri < 4; ++ri) {
                        if (q0 + dq >= pieces) continue;
                        uint32_t *x = w[dq][ri];
                        vmax = __vmaxu2(vmax, abs_max4(x[0], x[1], x[2], x[3]));
#pragma unroll
                        for (int i = 0; i < 4; ++i) x[i] = pack_f16x2(bf16_lo(x[i]), bf16_hi(x[i]));
                        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(adr[dq][ri]), "r"(x[0]), "r"(x[1]),
                                     "r"(x[2]), "r"(x[3])
                                     : "memory");
                    }
            }
            if (ones_col) {
                const int c = (D & 31) >> 3;
                const uint32_t base = vt + (uint32_t)(D >> 5) * 8192u + (uint32_t)((D & 7) * 2);
#pragma unroll
                for (int r = lane; r < kKeys; r += 32)
                    asm volatile("st.shared.u16 [%0], %1;" ::"r"(base + (uint32_t)r * 64u + (uint32_t)((c ^ ((r >> 1) & 3)) << 4)),
                                 "h"((unsigned short)0x3C00)
                                 : "memory");
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_VREADY + s));
            return true;
        };
        for (int j = 0; j < NB; ++j)
            if (!prep(j)) break;
        if ((vmax & 0xFFFFu) >= 0x4780u || (vmax >> 16) >= 0x4780u) record_status(kStatusRange);
    } else if (warp >= kSoftmaxWarp0) {
        // ------------------------------- softmax / epilogue ---------------------------
        // 8 warps: tile X = (warp - 4) / 4, lane quarter = warp % 4, one thread per query
        // row (its TMEM lane), all 128 keys of a block in its registers.
        const int sw = warp - kSoftmaxWarp0;
        const int X = sw >> 2;
        const int quarter = warp & 3;                     // TMEM lanes 32*quarter ..
        const int row = quarter * 32 + lane;              // query row of this thread in its tile
        const uint32_t lane_bits = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_col = tmem + lane_bits + TM::s(X);
        const uint32_t p_col = tmem + lane_bits + TM::p(X);
        const uint32_t o_col = tmem + lane_bits + TM::o(X);
        // this row of P_X in shared memory (box c adds c * 8 KB): 8-row groups 512 B apart,
        // 64-byte rows whose four 16-byte pieces are swizzled by (row >> 1) & 3
        const uint32_t p_row = sb + L.p0 + (uint32_t)X * 32768u + (uint32_t)(row >> 3) * 512u + (uint32_t)(row & 7) * 64u;
        const uint32_t p_swz = (uint32_t)((row >> 1) & 3);
        const float neg_inf = __int_as_float(0xff800000);
        const float scale = p.scale_log2;
        float m_used = neg_inf;     // max (log2 units) the probabilities are taken against
        float l_sum = 0.f;         // row sum, kept only when there is no padding column
        bool ok = true;
        for (int j = 0; ok && j < NB; ++j) {
            const int kb = j % p.nkb;
            const int valid = min(kKeys, p.HW - kb * kKeys);   // valid keys of this block
            if (!warp_wait(bar(B_SFULL + X), j & 1, 221, abort_flag)) { ok = false; break; }
            tc_fence_after();
            // the block's 128 scores into registers; then the score region is free
            uint32_t sr[128];
            tmem_ld128(s_col, sr);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SFREE + X));
            float m8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) m8[i] = neg_inf;
            if (valid >= kKeys) {
                // 8 independent chains, two scores per three-input max
#pragma unroll
                for (int i = 0; i < kKeys; i += 16)
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        m8[c] = fmax3(m8[c], __uint_as_float(sr[i + c]), __uint_as_float(sr[i + 8 + c]));
            } else {
#pragma unroll
                for (int i = 0; i < kKeys; ++i)
                    if (i < valid) m8[i & 7] = fmaxf(m8[i & 7], __uint_as_float(sr[i]));
            }
            const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])) * scale;
            float alpha = 1.f;
            const bool upd = mx > m_used + kLazyRescale;
            if (upd) {
                alpha = ex2(m_used - mx);
                m_used = mx;
            }
            if (j > 0 && __any_sync(0xffffffffu, upd)) {
                // the previous block's P V must be done accumulating before O is rescaled
                if (!warp_wait(bar(B_ODONE + X), (j - 1) & 1, 228, abort_flag)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < DP / 16; ++c) {
                    if (16 * c >= dpv) break;
                    uint32_t o[16];
                    const uint32_t a = o_col + (uint32_t)(16 * c);
                    tmem_ld16(a, o);
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st16(a, o);
                }
            }
            l_sum *= alpha;
            // probabilities from the registers as bf16 pairs, handed to the issuer one chunk
            // of 32 keys at a time
            const float neg_m = -m_used;
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                // all 32 exponentials of the chunk first, so that a warp keeps many in
                // flight on the exponential unit, then the bf16 packing
                float e[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) e[i] = ex2(fmaf(__uint_as_float(sr[32 * c + i]), scale, neg_m));
                if (valid < kKeys) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (32 * c + i >= valid) e[i] = 0.f;
                }
                uint32_t w[16];
                float ls = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    w[i] = pack_f16x2(e[2 * i], e[2 * i + 1]);
                    if (!ones_col) ls += e[2 * i] + e[2 * i + 1];
                }
                l_sum += ls;
                if constexpr (kPSmem) {
                    // keys 32c.. -> box c of P_X; this tile's P V of the previous block must be
                    // done reading P_X before its first chunk is overwritten (the block's
                    // completion barrier, which the rescale above also waits on)
                    if (c == 0 && j > 0 && !warp_wait(bar(B_ODONE + X), (j - 1) & 1, 229, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a = p_row + (uint32_t)c * 8192u;
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a + (((uint32_t)q ^ p_swz) << 4)),
                                     "r"(w[4 * q]), "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                                     : "memory");
                    if (c == kChunks - 1) {
                        // one proxy fence for the block (a fence per chunk measured 29.5 us
                        // per launch against 24.3), then the block goes to the issuer
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(B_PFULL + kChunks * X));
                    }
                } else {
                    // P over S (keys 32c.. -> TMEM columns 16c..): a chunk's store completes
                    // while the next chunk's exponentials run, then it is handed over
                    if (c > 0) {
                        tmem_st_wait();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(B_PFULL + kChunks * X + c - 1));
                    }
                    tmem_st16(p_col + (uint32_t)(16 * c), w);
                }
            }
            if (!ok) break;
            if constexpr (!kPSmem) {
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_PFULL + kChunks * X + kChunks - 1));
            }
        }
        // ---- epilogue: O / l -> bf16 rows staged in the tile's (now unused) Q buffer,
        //      then one TMA store of the warp's 32 rows -----------------------------------
        if (ok && warp_wait(bar(B_ODONE + X), (NB - 1) & 1, 224, abort_flag)) {
            tc_fence_after();
            float l = l_sum;
            if (ones_col) {
                uint32_t o[16];
                tmem_ld16(o_col + 16 * (p.D >> 4), o);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (i == (p.D & 15)) l = __uint_as_float(o[i]);
            }
            const float inv = 1.f / l;
            uint8_t *orow = sgen + L.q0 + X * TB + (size_t)row * (size_t)(p.D * 2);
#pragma unroll
            for (int c = 0; c < DP / 16; ++c) {
                if (16 * c >= dpv) break;
                uint32_t o[16];
                tmem_ld16(o_col + (uint32_t)(16 * c), o);
#pragma unroll
                for (int hlf = 0; hlf < 2; ++hlf) {
                    const int col = 16 * c + 8 * hlf;
                    if (col < p.D) {
                        auto v = [&](int i) { return __uint_as_float(o[8 * hlf + i]) * inv; };
                        uint4 w;
                        w.x = pack_bf16x2(v(0), v(1));
                        w.y = pack_bf16x2(v(2), v(3));
                        w.z = pack_bf16x2(v(4), v(5));
                        w.w = pack_bf16x2(v(6), v(7));
                        *reinterpret_cast<uint4 *>(orow + 2 * col) = w;
                    }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            // rows past HW are not written by the TMA unit; a box starting past HW is skipped
            const int r0 = row0 + X * kRows + quarter * 32;
            if (lane == 0 && r0 < p.HW) {
                tma_store_4d(&tm.o, sb + L.q0 + X * TB + (uint32_t)(quarter * 32 * p.D * 2), 0, h, r0,
                             b * p.n + f);
                bulk_commit();
                bulk_wait_read<0>();
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

// Dynamic shared memory is never below this, so at most one CTA is resident per SM and the
// 512-column TMEM allocation never waits on another CTA.
constexpr uint32_t kMinSmem = 116 * 1024;

uint32_t spatial_smem_bytes(int D)
{
    const uint32_t s = spatial_layout((D + 15) / 16).total;
    return s < kMinSmem ? kMinSmem : s;
}

template <int NKD>
static cudaError_t launch_nkd(const SpatialMaps &m, const SpatialParams &p, cudaStream_t stream)
{
    constexpr uint32_t smem = spatial_layout(NKD).total < kMinSmem ? kMinSmem : spatial_layout(NKD).total;
    static std::atomic<uint64_t> configured{0};
    const cudaError_t e =
        ensure_smem_attr(configured, reinterpret_cast<const void *>(&k_spatial_prefix<NKD>), (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(p.B * p.n * p.H * p.q_pairs);
    return launch_chained(k_spatial_prefix<NKD>, dim3(grid), dim3(kThreads), smem, stream, m, p);
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
