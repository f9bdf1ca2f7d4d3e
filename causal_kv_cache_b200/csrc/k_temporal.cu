// k_temporal.cu -- causal temporal attention over the cached prefix queue (sm_100a).
//
// Ca2-VDM ("Ca2-VDM" papernotes page, 关键设计 1, equation CausalAttn): per spatial token
// and head, the l queries of the current chunk attend to the P_k queued clean-prefix
// frames followed by the chunk's own frames 0..c -- the chunk's rows of
// Softmax(QK^T/sqrt(D) + M)V with M_ij = -inf for i < j.  Every queued frame is visible
// to every chunk query, so the queued keys form a set: the kernel visits ring slots in
// physical order 0..Pmax-1 and masks slots that hold no queued frame, which makes every
// ring read one contiguous run.  Only the chunk's own keys carry the causal mask.
//
// Design (HBM-bound: each cached K/V byte is read once per call):
//   * Temporal tensors are token-major: the chunk is [B][HW][n][H][D]; the ring is
//     [B][HW][H][Pmax][D], head-major within a token, so one (token, head) history is one
//     contiguous run (41 x 144 B at the Open-Sora shape).
//   * Work item = (video b, token s, group of G heads).  A stage holds 16 key frames of
//     the G heads, in shared memory as [head][frame][D]: each head's 16 key rows are
//     consecutive 2*D-byte rows (an odd number of 16-byte units for D = 72, so ldmatrix is
//     bank-conflict free).
//   * Stage 0 is the chunk's own 16 frames, one TMA box per tensor viewed 5-D (head dim,
//     frame, head, token, video); frames past n are zero-filled by the TMA unit.  Stage 0
//     holds chunk frame 0, which every query sees, so the running max is finite from the
//     first stage on.  Then the ring in 16-slot groups: per head one bulk copy of the
//     group's consecutive slots (2304 B for a full group; contiguous copies of this size
//     stream at the HBM rate, where boxes of 144-byte rows measured well below it).
//     Groups with no queued slot are skipped (host-computed mask).
//   * Work distribution: one CTA per work item in the grid; a resident CTA finishes its
//     own item and then takes over the items of CTAs that have not started yet (cluster
//     launch control), so every SM stays busy to the end whatever its share of items.
//     One producer warp keeps NS stages of K and V in flight on mbarriers and runs ahead
//     across items; G consumer warps (one head each) compute.
//   * Per head the contraction is tiny (8 queries x 16 keys per stage x D), so both
//     products use mma.sync on registers: S^T = K Q^T (keys on M, the 8 queries on N),
//     then O^T += V^T P^T.  Each lane owns the same two query columns in both
//     accumulators, so the online-softmax rescale is lane-local; movmatrix turns P^T
//     into the B operand and O^T back into rows for the stores.  P V runs in fp16 (P with
//     11 significant bits rather than bf16's 8): the ring keeps V in fp16 (converted
//     exactly when written), and the chunk's own V is converted in registers.  The
//     reference max of the exponentials moves
//     only when a score exceeds it by more than 2^8 (one warp vote per stage; the max
//     reduction and the rescale run only then), which leaves each softmax row unchanged
//     after normalisation.
//   * Ring rows that hold no queued frame are masked, and their V rows are zero, so stale
//     bits (of the caller's buffer or of an earlier stage) never reach the accumulator.
//     The producer zeroes the V rows past Pmax, which the ring copy does not write, before
//     it arms the stage (off the consumers' path), so the consumers write shared memory
//     (and fence it against the next copy into the stage) only for slots inside Pmax that
//     hold no queued frame, which happens only while the queue fills.
#include <atomic>
#include <cstdint>
#include <cuda_bf16.h>

#include "ca2_device.cuh"
#include "ca2_kernels.h"

namespace ca2 {

namespace {

constexpr int kStages = 4;       // K+V stages in flight per CTA
constexpr int kKeys = 16;        // key frames per stage
constexpr int kQ = 8;            // queries per (token, head): the mma N extent
constexpr float kLazy = 8.0f;    // log2 units
constexpr int kPrefetchCtas = 128;   // CTAs that prefetch ring runs into L2 before the dependency wait
constexpr int kPrefetchItems = 4;    // consecutive items each of them covers

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
__device__ __forceinline__ void mma16816_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// bf16 pair -> fp16 pair (exact within the fp16 range)
__device__ __forceinline__ uint32_t bf2_to_h2(uint32_t w) { return pack_f16x2(bf16_lo(w), bf16_hi(w)); }
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
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const void *tmap, int c0, int c1, int c2, int c3, int c4,
                                            uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
        "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
        : "memory");
}

struct Layout {
    uint32_t kv_box;        // bytes of one K (or V) box: G heads x 16 frames x D
    uint32_t stage_bytes;   // K box then V box
    uint32_t q_box;         // G heads x 8 frames x D
    uint32_t q_off, bar_off, misc_off, total;
};

__host__ __device__ inline Layout make_layout(int G, int D)
{
    Layout L;
    L.kv_box = (uint32_t)(G * kKeys * D * 2);
    L.stage_bytes = 2u * L.kv_box;
    L.q_box = (uint32_t)(G * kQ * D * 2);
    L.q_off = kStages * L.stage_bytes;
    L.bar_off = (L.q_off + 2u * L.q_box + 7u) & ~7u;
    // after the barriers: the 16-byte work-request response, the abort flag, two item ids
    L.misc_off = (L.bar_off + 8u * (2 * kStages + 5) + 15u) & ~15u;
    L.total = L.misc_off + 32u;
    return L;
}

}  // namespace

template <int DT>
__global__ void __launch_bounds__(32 * (kMaxTemporalGroup + 1))
    k_temporal_causal(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const TemporalParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = p.G;
    const int D = p.D;
    const Layout L = make_layout(G, D);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L.bar_off;
    auto full_bar = [&](int i) { return bar0 + 8u * i; };
    auto empty_bar = [&](int i) { return bar0 + 8u * (kStages + i); };
    auto qfull_bar = [&](int i) { return bar0 + 8u * (2 * kStages + i); };
    auto qempty_bar = [&](int i) { return bar0 + 8u * (2 * kStages + 2 + i); };
    auto work_bar = [&]() { return bar0 + 8u * (2 * kStages + 4); };
    const uint32_t work_resp = sbase + L.misc_off;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc_off + 16u);
    volatile int *item_ids = reinterpret_cast<volatile int *>(smem + L.misc_off + 20u);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(full_bar(i), 1);
            mbar_init(empty_bar(i), G);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(qfull_bar(i), 1);
            mbar_init(qempty_bar(i), G);
        }
        mbar_init(work_bar(), 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    __syncthreads();
    const int groups = p.H / G;
    // Before waiting for the previous kernel, the first kPrefetchCtas CTAs (the first
    // launched, so the ones that start while the previous kernel still runs) ask L2 for the
    // ring runs of the items the first wave will take: kPrefetchItems consecutive items each.
    // The ring is cache state, and a prefetch only moves data into L2, so this is safe
    // whatever the previous kernel writes; the copies after the wait then read L2 instead of
    // HBM while the previous kernel, if it is compute-bound, leaves HBM idle.
    if (warp == G && (int)blockIdx.x < kPrefetchCtas && p.ring_box_mask) {
        const int n_ring_runs = __popc(p.ring_box_mask) * 2 * G;     // (group, tensor, head) runs
        const int first = (int)blockIdx.x * kPrefetchItems;
        for (int t = lane; t < kPrefetchItems * n_ring_runs; t += 32) {
            const int it = first + t / n_ring_runs;
            if (it >= p.n_items) break;
            int r = t % n_ring_runs;
            const int w = r % G;
            const int kv = (r / G) & 1;
            int k = r / (2 * G);                                 // k-th set bit of the mask
            uint32_t mask = p.ring_box_mask;
            for (; k > 0; --k) mask &= mask - 1;
            const int box = __ffs(mask) - 1;
            const int hg = it % groups;
            const int s = (it / groups) % p.HW;
            const int b = it / (groups * p.HW);
            const int s0 = box * kKeys;
            const int ns = min(kKeys, p.Pmax - s0);
            const size_t off = ((((size_t)b * p.HW + (size_t)s) * (size_t)p.H + (size_t)(hg * G + w)) *
                                    (size_t)p.Pmax + (size_t)s0) * ((size_t)D * 2u);
            if (CA2_IN_BOUNDS(off + (size_t)ns * D * 2 <= (size_t)p.ring_bytes, 14))
                bulk_prefetch_l2((kv ? p.rv : p.rk) + off, (uint32_t)(ns * D * 2));
        }
    }
    // the previous kernel on the stream has completed: inputs may now be read
    wait_previous_kernel();
    allow_next_kernel();

    // stage list: stage 0 = the chunk's frames, then the ring boxes whose bit is set
    const int n_ring = __popc(p.ring_box_mask);
    const int n_stages = 1 + n_ring;

    if (warp == G) {
        // ------------------------------ producer ------------------------------------
        // The whole warp runs the loop (warp-uniform waits); lane 0 issues the TMA boxes and
        // the work requests, and the ring copies of a stage go out in one warp instruction,
        // lane i < 2G issuing one head's K (i < G) or V run: a single issuing thread was
        // measured at ~150 cycles per bulk copy.
        // Work items: this CTA's own index first, then items of CTAs of the grid that
        // have not started yet, taken over through cluster launch control until none is
        // left; every SM stays busy until the last items, whatever their count per SM.
        int stage = 0, li = 0;
        int requests = 0;           // work requests made (phases of work_bar)
        bool can_take = true;       // no request has failed yet
        bool pending = false;       // a request whose response has not been read
        bool ok = true;
        int it = blockIdx.x;
        while (ok && it >= 0 && it < p.n_items) {
            const int hg = it % groups;
            const int s = (it / groups) % p.HW;
            const int b = it / (groups * p.HW);
            const int qs = li & 1;
            if (li >= 2 && !warp_wait(qempty_bar(qs), ((li - 2) >> 1) & 1, 101, abort_flag)) { ok = false; break; }
            if (lane == 0) {
                item_ids[qs] = it;
                mbar_expect_tx(qfull_bar(qs), L.q_box);
                tma_load_5d(sbase + L.q_off + (uint32_t)qs * L.q_box, &tm_q, 0, 0, hg * G, s, b, qfull_bar(qs));
            }
            ++li;
            uint32_t mask = p.ring_box_mask;
            for (int st = 0; st < n_stages; ++st, ++stage) {
                const int slot = stage % kStages;
                if (stage >= kStages &&
                    !warp_wait(empty_bar(slot), ((stage / kStages) - 1) & 1, 102, abort_flag)) { ok = false; break; }
                const uint32_t dst = sbase + (uint32_t)slot * L.stage_bytes;
                if (st == 0) {
                    if (lane == 0) {
                        mbar_expect_tx(full_bar(slot), L.stage_bytes);
                        tma_load_5d(dst, &tm_k, 0, 0, hg * G, s, b, full_bar(slot));
                        tma_load_5d(dst + L.kv_box, &tm_v, 0, 0, hg * G, s, b, full_bar(slot));
                    }
                } else {
                    // ring slots [16 box, 16 box + ns): one contiguous run of ns rows per
                    // head and tensor (the ring is head-major within a token)
                    const int box = __ffs(mask) - 1;
                    mask &= mask - 1;
                    const int s0 = box * kKeys;
                    const int ns = min(kKeys, p.Pmax - s0);
                    const uint32_t run = (uint32_t)(ns * D * 2);
                    if (ns < kKeys) {
                        // V rows ns..15 of every head := 0 (generic-proxy writes, ordered before
                        // the stage's arrive and before any later copy into the stage)
                        const uint32_t pad16 = (uint32_t)((kKeys - ns) * D * 2) / 16u;
                        for (uint32_t i = (uint32_t)lane; i < (uint32_t)G * pad16; i += 32u) {
                            const uint32_t w = i / pad16;
                            const uint32_t a = dst + L.kv_box + w * (uint32_t)(kKeys * D * 2) + run + 16u * (i - w * pad16);
                            asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};" ::"r"(a), "r"(0u) : "memory");
                        }
                        fence_proxy_async_smem();
                    }
                    __syncwarp();
                    if (lane == 0) mbar_expect_tx(full_bar(slot), 2u * (uint32_t)G * run);
                    __syncwarp();
                    if (lane < 2 * G) {
                        const int w = lane % G;
                        const int kv = lane / G;
                        const size_t off = ((((size_t)b * p.HW + (size_t)s) * (size_t)p.H + (size_t)(hg * G + w)) *
                                                (size_t)p.Pmax + (size_t)s0) * ((size_t)D * 2u);
                        // (a skipped copy leaves the stage's barrier short: the consumers' bounded
                        // wait then gives up, after the bounds record)
                        if (CA2_IN_BOUNDS(off + run <= (size_t)p.ring_bytes, 11))
                            bulk_g2s(dst + (uint32_t)kv * L.kv_box + (uint32_t)(w * kKeys * D * 2),
                                     (kv ? p.rv : p.rk) + off, run, full_bar(slot));
                    }
                }
            }
            if (!ok) break;
            // claim the next item only once a ring slot is free for its first stage: a claim
            // made earlier would reserve it long before this CTA can start on it, and the
            // CTAs holding one more item at the end of the list set the tail
            int next = -1;
            if (can_take) {
                if (stage >= kStages &&
                    !warp_wait(empty_bar(stage % kStages), ((stage / kStages) - 1) & 1, 102, abort_flag)) { ok = false; break; }
                if (lane == 0) {
                    mbar_expect_tx(work_bar(), 16u);
                    work_request(work_resp, work_bar());
                }
                pending = true;
            }
            if (pending) {
                if (!warp_wait(work_bar(), requests & 1, 105, abort_flag)) { ok = false; break; }
                ++requests;
                pending = false;
                uint32_t x;
                if (work_response(work_resp, x)) next = (int)x;
                else can_take = false;
            }
            it = next;
        }
        if (lane == 0) {
            // no further item: a sentinel in the next Q slot ends the consumers' loop
            if (ok) {
                const int qs = li & 1;
                if (li < 2 || mbar_wait(qempty_bar(qs), ((li - 2) >> 1) & 1, 101, abort_flag)) {
                    item_ids[qs] = -1;
                    mbar_arrive(qfull_bar(qs));
                }
            }
            // an unanswered request still writes shared memory: wait for it (bounded)
            if (pending) mbar_wait(work_bar(), requests & 1, 0, nullptr, 2000000ull);
            // wind-down after an abort: let the loads still in flight land before exiting
            // (each slot's last use is the most recent phase of its barrier)
            if (!ok) {
                for (int k = stage - 1; k >= 0 && k >= stage - kStages; --k)
                    mbar_wait(full_bar(k % kStages), (k / kStages) & 1, 0, nullptr, 2000000ull);
                for (int k = li - 1; k >= 0 && k >= li - 2; --k)
                    mbar_wait(qfull_bar(k & 1), (k >> 1) & 1, 0, nullptr, 2000000ull);
            }
        }
    } else if (warp < G) {
        // ------------------------------ consumers -----------------------------------
        const int w = warp;
        const uint32_t head_kv = (uint32_t)(w * kKeys * D * 2);   // this head's rows in a K/V box
        const uint32_t head_q = (uint32_t)(w * kQ * D * 2);
        const uint32_t row = (uint32_t)(D * 2);                   // bytes per key/query row
        const int q0 = 2 * (lane & 3);        // this lane's two query columns: q0, q0 + 1
        const int krow = lane >> 2;            // this lane's key rows in a stage: krow, krow + 8
        const float neg_inf = __int_as_float(0xff800000);
        uint32_t vmax = 0;                     // per-half max of |v| bits of the chunk's V
        int stage = 0;
        for (int li = 0;; ++li) {
            const int qs = li & 1;
            if (!warp_wait(qfull_bar(qs), (li >> 1) & 1, 103, abort_flag)) break;
            const int it = item_ids[qs];      // written before the Q slot's barrier arrive
            if (it < 0) break;
            const int hg = it % groups;
            const int s = (it / groups) % p.HW;
            const int b = it / (groups * p.HW);

            // Q as the B operand (col-major K x N = dims x queries == Q rows [query][dim])
            uint32_t qb[DT][2];
            {
                const uint32_t qbase = sbase + L.q_off + (uint32_t)qs * L.q_box + head_q;
#pragma unroll
                for (int kk = 0; kk < DT; ++kk) {
                    if (16 * kk + 16 <= D) {
                        ldsm_x2(qbase + (uint32_t)(lane & 7) * row + (uint32_t)(16 * kk + 8 * ((lane >> 3) & 1)) * 2u,
                                qb[kk][0], qb[kk][1]);
                    } else {
                        ldsm_x1(qbase + (uint32_t)(lane & 7) * row + (uint32_t)(16 * kk) * 2u, qb[kk][0]);
                        qb[kk][1] = 0u;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(qempty_bar(qs));

            float m_run[2] = {neg_inf, neg_inf};
            float l_part[2] = {0.f, 0.f};
            float acc[DT][4];
#pragma unroll
            for (int t = 0; t < DT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

            bool ok = true;
            uint32_t mask = p.ring_box_mask;
            for (int st = 0; st < n_stages; ++st, ++stage) {
                const int slot = stage % kStages;
                // key rows of this stage: visibility per (row, query column)
                bool vis[2][2];
                bool zero_v = false;
                if (st == 0) {
                    vis[0][0] = krow < p.n && krow <= q0;
                    vis[0][1] = krow < p.n && krow <= q0 + 1;
                    vis[1][0] = vis[1][1] = false;      // chunk frames 8..15 do not exist
                } else {
                    const int box = __ffs(mask) - 1;
                    mask &= mask - 1;
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const int sl = box * kKeys + krow + 8 * hr;
                        int age = sl - p.head;
                        if (age < 0) age += p.Pmax;
                        const bool v = sl < p.Pmax && age < p.Pk;
                        vis[hr][0] = vis[hr][1] = v;
                    }
                    // slots inside Pmax that hold no queued frame: zero their V rows (the
                    // producer has zeroed the rows past Pmax)
                    const int sl = box * kKeys + (lane & 15);
                    int age = sl - p.head;
                    if (age < 0) age += p.Pmax;
                    zero_v = sl < p.Pmax && age >= p.Pk;
                }
                if (!warp_wait(full_bar(slot), (stage / kStages) & 1, 104, abort_flag)) { ok = false; break; }
                const uint32_t kbase = sbase + (uint32_t)slot * L.stage_bytes + head_kv;
                const uint32_t vbase = kbase + L.kv_box;
                if (__any_sync(0xffffffffu, zero_v)) {
                    if (zero_v && lane < 16) {
                        const uint32_t r0 = vbase + (uint32_t)lane * row;
                        for (int o = 0; o < D * 2; o += 16)
                            asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};" ::"r"(r0 + o), "r"(0u) : "memory");
                        // these generic-proxy writes must be ordered before the next copy
                        // into this stage
                        fence_proxy_async_smem();
                    }
                    __syncwarp();
                }

                // S^T = K Q^T : 16 keys x 8 queries
                float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < DT; ++kk) {
                    const uint32_t a = kbase + (uint32_t)((lane & 7) + 8 * ((lane >> 3) & 1)) * row;
                    if (16 * kk + 16 <= D) {
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4(a + (uint32_t)(16 * kk + 8 * (lane >> 4)) * 2u, a0, a1, a2, a3);
                        mma16816(c, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
                    } else {
                        uint32_t a0, a1;
                        ldsm_x2(a + (uint32_t)(16 * kk) * 2u, a0, a1);
                        mma1688(c, a0, a1, qb[kk][0]);
                    }
                }
                float sc[4];
                sc[0] = vis[0][0] ? c[0] * p.scale_log2 : neg_inf;
                sc[1] = vis[0][1] ? c[1] * p.scale_log2 : neg_inf;
                sc[2] = vis[1][0] ? c[2] * p.scale_log2 : neg_inf;
                sc[3] = vis[1][1] ? c[3] * p.scale_log2 : neg_inf;
                float mx0 = fmaxf(sc[0], sc[2]);
                float mx1 = fmaxf(sc[1], sc[3]);
                // the reference max moves only when a score exceeds it by more than 2^8 (always
                // on stage 0, which holds chunk frame 0, visible to every query)
                if (__any_sync(0xffffffffu, mx0 > m_run[0] + kLazy || mx1 > m_run[1] + kLazy)) {
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1) {
                        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                    }
                    const float mn0 = fmaxf(m_run[0], mx0);
                    const float mn1 = fmaxf(m_run[1], mx1);
                    const float al0 = ex2(m_run[0] - mn0);
                    const float al1 = ex2(m_run[1] - mn1);
                    m_run[0] = mn0;
                    m_run[1] = mn1;
                    l_part[0] *= al0;
                    l_part[1] *= al1;
#pragma unroll
                    for (int t = 0; t < DT; ++t) {
                        acc[t][0] *= al0;
                        acc[t][1] *= al1;
                        acc[t][2] *= al0;
                        acc[t][3] *= al1;
                    }
                }
                // probabilities in fp16 (11 significant bits; bf16 P would carry up to 2^-9
                // relative error into every output, the order of the output's own rounding);
                // the normaliser sums the fp32 values (2^-12 from the rounded ones)
                const float e0 = ex2(sc[0] - m_run[0]), e1 = ex2(sc[1] - m_run[1]);
                const float e2 = ex2(sc[2] - m_run[0]), e3 = ex2(sc[3] - m_run[1]);
                l_part[0] += e0 + e2;
                l_part[1] += e1 + e3;
                const uint32_t pb0 = movm_t(pack_f16x2(e0, e1));
                const uint32_t pb1 = movm_t(pack_f16x2(e2, e3));
                // O^T += V^T P^T, 16 head dims per m-tile
#pragma unroll
                for (int t = 0; t < DT; ++t) {
                    if (16 * t + 16 <= D) {
                        const int j = lane >> 3;
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4_t(vbase + (uint32_t)((lane & 7) + 8 * (j >> 1)) * row + (uint32_t)(16 * t + 8 * (j & 1)) * 2u,
                                  a0, a1, a2, a3);
                        if (st == 0) {
                            // the chunk's own V arrives as bf16; its key rows 8..15 (a2, a3) are
                            // frames past the chunk (n <= 8), zero-filled, the same in fp16
                            vmax = __vmaxu2(vmax, abs_max4(a0, a1, 0u, 0u));
                            a0 = bf2_to_h2(a0), a1 = bf2_to_h2(a1);
                        }
                        mma16816_f16(acc[t], a0, a1, a2, a3, pb0, pb1);
                    } else {
                        uint32_t a0, a2;
                        ldsm_x2_t(vbase + (uint32_t)((lane & 7) + 8 * ((lane >> 3) & 1)) * row + (uint32_t)(16 * t) * 2u,
                                  a0, a2);
                        if (st == 0) {
                            vmax = __vmaxu2(vmax, abs_max4(a0, 0u, 0u, 0u));
                            a0 = bf2_to_h2(a0);
                        }
                        mma16816_f16(acc[t], a0, 0u, a2, 0u, pb0, pb1);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(slot));
            }
            if (!ok) break;

            // normalise; transpose O^T back to rows with movmatrix; each lane stores two
            // 4-byte pieces of its query row
            float l0 = l_part[0], l1 = l_part[1];
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l0 += __shfl_xor_sync(0xffffffffu, l0, off);
                l1 += __shfl_xor_sync(0xffffffffu, l1, off);
            }
            const float i0 = 1.f / l0, i1 = 1.f / l1;
            const int qrow = lane >> 2;
            const long long o0 = (((long long)b * p.HW + s) * p.n + qrow) * p.pitch +
                                 (long long)(hg * G + w) * D + 2 * (lane & 3);
            __nv_bfloat16 *orow = p.out + o0;
#pragma unroll
            for (int t = 0; t < DT; ++t) {
                const uint32_t y0 = movm_t(pack_bf16x2(acc[t][0] * i0, acc[t][1] * i1));
                if (qrow < p.n && CA2_IN_BOUNDS(o0 + 16 * t + 2 <= p.out_elems, 12))
                    *reinterpret_cast<uint32_t *>(orow + 16 * t) = y0;
                if (16 * t + 16 <= D) {
                    const uint32_t y1 = movm_t(pack_bf16x2(acc[t][2] * i0, acc[t][3] * i1));
                    if (qrow < p.n && CA2_IN_BOUNDS(o0 + 16 * t + 10 <= p.out_elems, 13))
                        *reinterpret_cast<uint32_t *>(orow + 16 * t + 8) = y1;
                }
            }
        }
        // a chunk V beyond the fp16 range (|v| >= 65536, inf, NaN): a range error
        if ((vmax & 0xFFFFu) >= 0x4780u || (vmax >> 16) >= 0x4780u) record_status(kStatusRange);
    }
}

// ---------------------------------------------------------------------------------------
uint32_t temporal_smem_bytes(int G, int D) { return make_layout(G, D).total; }

template <int DT>
static cudaError_t launch_dt(const TemporalMaps &m, const TemporalParams &p, int grid, cudaStream_t stream)
{
    const uint32_t smem = make_layout(p.G, p.D).total;
    static std::atomic<uint64_t> configured{0};
    const cudaError_t e = ensure_smem_attr(configured, reinterpret_cast<const void *>(&k_temporal_causal<DT>),
                                           (int)make_layout(kMaxTemporalGroup, 16 * DT).total);
    if (e != cudaSuccess) return e;
    return launch_chained(k_temporal_causal<DT>, dim3(grid), dim3(32 * (p.G + 1)), smem, stream, m.q, m.k, m.v, p);
}

cudaError_t launch_temporal(const TemporalMaps &m, const TemporalParams &p, int grid, cudaStream_t stream)
{
    switch ((p.D + 15) / 16) {
    case 1: return launch_dt<1>(m, p, grid, stream);
    case 2: return launch_dt<2>(m, p, grid, stream);
    case 3: return launch_dt<3>(m, p, grid, stream);
    case 4: return launch_dt<4>(m, p, grid, stream);
    case 5: return launch_dt<5>(m, p, grid, stream);
    case 6: return launch_dt<6>(m, p, grid, stream);
    case 7: return launch_dt<7>(m, p, grid, stream);
    case 8: return launch_dt<8>(m, p, grid, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ca2
