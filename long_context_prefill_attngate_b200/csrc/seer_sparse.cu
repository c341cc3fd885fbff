// seer_sparse.cu — block-sparse causal attention prefill for sm_100a with one
// query head's query block per tile (no union of several heads' key lists).
//
// What it computes ("Learning Intrinsic Sparse Attention in Your LLMs",
// rebuttal Weakness 5, the inference kernel): for each (head, query block)
// an online softmax over that row's selected key blocks only, token-causal
// inside the diagonal block.  The mask is compacted on the fly into the row's
// ascending list of key blocks, so a skipped block costs no load and no MMA.
//
// B200 design:
//  * A tile is 64 query rows of one head, so the MMA rows all want the same
//    key blocks and no work is spent on blocks another head selected.  M = 64
//    tcgen05.mma runs at half the M = 128 rate, so the key side is made wide
//    instead: each step takes TWO selected key blocks, S = Q K^T with N = 128
//    (and O += P V with K = 128 keys, N = d).  A row with an odd count ends with
//    a single-block step (N = 64, K = 64), so nothing is padded.
//  * TMEM: three S buffers (128 fp32 columns each) and one O (128).  P(t)
//    (packed bf16) overwrites the first 64 columns of S buffer t % 3 and PV
//    reads it from there as a TS MMA.  S(t) is issued once PV(t - 3) has
//    completed, so S runs two steps ahead of the softmax: the softmax of a step
//    has about two steps of tensor-pipe time before its P is needed.  M = 64
//    rows live in lanes 32 (m / 16) + m % 16.
//  * Softmax: two groups of four warps take alternate steps (group = step % 2),
//    one warp per TMEM lane quarter.  With the 16x32bx2 load shape thread c of a
//    warp holds key block c of the step (64 scores in registers), so a row's
//    max is one shuffle; the running max is handed from one group to the other
//    through shared memory (one mbarrier per lane quarter).  The two groups'
//    exponentials fall in different phases, so they share the SFU instead of
//    colliding on it, and no warp waits for a partner within a step.  The
//    running max moves only when it grows by more than 2^8 (log2 domain): P
//    stays <= 256 and the O rescale (a TMEM round trip) is rare.  Each group
//    keeps its own row sum, rescaled when it sees the max move; the two sums
//    meet in the epilogue.
//  * Two MMA-issuing threads: one issues the S MMAs, the other the PV MMAs.
//    A tcgen05.mma issue blocks at the tensor pipe's rate and every commit or
//    barrier check of the issuing thread is serial latency; with two issuers
//    one thread's checks are covered by the other's MMAs.
//  * K and V rings of two stages (one step's two key blocks each): a stage is
//    free once the S (or PV) MMA of the step two back has completed, which the
//    s_full (pv_done) commit already signals.  A TMA instruction holds its issuing
//    thread for a long time and one thread's copies complete roughly one after
//    another, so every box of a stage is issued by its own lane.
//  * Warps: 0-7 softmax and epilogue (a tile's O -> bf16 -> global and LSE are
//    read out by the group that takes the next step, right after its P store,
//    and the next tile's first PV waits for that), 8 TMA for Q and K, 9 S
//    issuer, 10 mask -> list builder, 11 TMA for V, 12 PV issuer.  One CTA per
//    SM, persistent, tiles taken from a launch-wide atomic counter in
//    KV-head-major order (concurrent tiles share one KV head's K/V in L2), the
//    longest causal rows first.
//  * K stage laid out [d panel][128 keys][128 B] so a single N = 128 descriptor
//    spans both blocks; V stage [block][d panel][64 keys][128 B] (MN-major B
//    operand).  Q is double-buffered across tiles.
//  * Every wait is bounded; a wait that runs out raises the device status word,
//    the CTA drains its in-flight copies and MMAs, frees TMEM and exits.
#include <cuda_bf16.h>

#include <type_traits>

#include "seer_internal.h"
#include "seer_ptx.cuh"


namespace seer {

namespace {

constexpr int kThreads = 416;         // 13 warps (four on one SM sub-partition: <= 128 registers)
constexpr uint64_t kDrain = 200000000ull;
constexpr int kGroupWarps = 4;        // softmax warps per group (one per lane quarter)
constexpr int kListConsumers = 12;    // Q/K and V producers, S and PV issuers, 8 softmax warps
constexpr int kWarpQK = 8, kWarpS = 9, kWarpList = 10, kWarpV = 11, kWarpPV = 12;
constexpr int kStepBlocks = 2;        // key blocks per step

struct TileInfo {
    int count, b, h, i, diag;
};

struct SParams {
    int B, Hq, Hkv, S, nb, g;
    long long n_units;
    float scale_log2;
    const uint8_t *mask;
    __nv_bfloat16 *o;
    float *lse;
    uint64_t timeout_ns;
    int *status;
    unsigned long long *tile_ctr;
    unsigned long long tile_base;
    int list_stride;
};

template <int D>
struct Geo {
    static constexpr int kPanels = D / 64;
    static constexpr int kQBytes = 64 * D * 2;        // one query block
    static constexpr int kBlkBytes = 64 * D * 2;      // one key block (K or V)
    static constexpr int kPair = 2 * kBlkBytes;       // a stage: two key blocks
    static constexpr int kNK = 2, kNV = 2;            // ring depths in stages (step n reuses step n - 2's)
    static constexpr int kQBufs = 2;                  // query-block buffers
    static constexpr int kOffK = kQBufs * kQBytes;
    static constexpr int kOffV = kOffK + kNK * kPair;
    static constexpr int kOffBar = kOffV + kNV * kPair;
    // s_full, p_full and pv_done cycle over the three S buffers (step % 3): S may
    // run two steps ahead of the softmax, and three slots keep every parity wait
    // unambiguous (S(t + 3) cannot complete before P(t) has been written).
    // m_ready[slot][quarter] hands the running max from one softmax group to the
    // other (slot = step % 2); l_ready[slot][quarter] collects both groups' row
    // sums of a tile (slot = tile % 2).
    static constexpr int kQFull = 0, kQEmpty = 2, kKFull = 4, kVFull = kKFull + kNK, kSFull = kVFull + kNV, kPFull = kSFull + 3, kPVDone = kPFull + 3,
                         kOFull = kPVDone + 3, kOFree = kOFull + 2, kListFull = kOFree + 2, kListEmpty = kListFull + 2,
                         kDrain = kListEmpty + 2, kMReady = kDrain + 2, kLReady = kMReady + 8, kNumBars = kLReady + 8;
    static constexpr int kOffM = kOffBar + kNumBars * 8;           // float [2 slots][64 rows]
    static constexpr int kOffL = kOffM + 2 * 64 * 4;               // float [2 slots][2 groups][2 (l, m)][64 rows]
    static constexpr int kOffInfo = kOffL + 2 * 2 * 2 * 64 * 4;
    static constexpr int kOffMisc = kOffInfo + 2 * (int)sizeof(TileInfo);
    static constexpr int kOffList = (kOffMisc + 16 + 15) / 16 * 16;
    static int list_stride(int nb) { return (nb + 7) / 8 * 8; }    // uint16 entries per buffer
    // Bytes the layout uses from its 1024-aligned base; the window asked for adds up
    // to 1 KB for aligning the base, as much of it as the 227 KB cap leaves (the
    // kernel checks that the aligned layout fits the window it got).
    static int smem_used(int nb) { return kOffList + 2 * list_stride(nb) * 2; }
    static int smem_bytes(int nb) { return smem_used(nb) + 1024 < 227 * 1024 ? smem_used(nb) + 1024 : 227 * 1024; }
};

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitCtx &w)
{
    const bool r = mbar_wait(bar, parity, w);
    return __all_sync(0xffffffffu, r);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const SParams p)
{
    using G = Geo<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase;
    const uint32_t sK = sbase + G::kOffK;
    const uint32_t sV = sbase + G::kOffV;
    const uint32_t sBar = sbase + G::kOffBar;
    auto bar = [&](int idx) -> uint32_t { return sBar + 8u * idx; };
    TileInfo *infos = reinterpret_cast<TileInfo *>(smem + G::kOffInfo);
    uint32_t *tmem_base_ptr = reinterpret_cast<uint32_t *>(smem + G::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + G::kOffMisc + 4);
    uint16_t *lists = reinterpret_cast<uint16_t *>(smem + G::kOffList);
    const WaitCtx wc{abort_flag, p.timeout_ns, p.status};
    const int lstride = p.list_stride;

    {   // the aligned layout must fit the dynamic window (uniform over the grid)
        uint32_t window;
        asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(window));
        const uint32_t pad = (uint32_t)(reinterpret_cast<uintptr_t>(smem) - reinterpret_cast<uintptr_t>(smem_raw));
        if (pad + (uint32_t)G::kOffList + 4u * (uint32_t)lstride > window) {
            if (threadIdx.x == 0)
                set_status(p.status, kStatusSmem);
            return;
        }
    }
    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar(G::kQFull + x), 1);
            mbar_init(bar(G::kQEmpty + x), 1);
            mbar_init(bar(G::kOFull + x), 1);
            mbar_init(bar(G::kOFree + x), kGroupWarps);
            mbar_init(bar(G::kListFull + x), 1);
            mbar_init(bar(G::kListEmpty + x), kListConsumers);
            mbar_init(bar(G::kDrain + x), 1);
        }
        for (int x = 0; x < G::kNK; ++x)
            mbar_init(bar(G::kKFull + x), 1);
        for (int x = 0; x < G::kNV; ++x)
            mbar_init(bar(G::kVFull + x), 1);
        for (int x = 0; x < 3; ++x) {
            mbar_init(bar(G::kSFull + x), 1);
            mbar_init(bar(G::kPFull + x), kGroupWarps);
            mbar_init(bar(G::kPVDone + x), 1);
        }
        for (int x = 0; x < 8; ++x) {
            mbar_init(bar(G::kMReady + x), 1);     // the publishing warp of the lane quarter
            mbar_init(bar(G::kLReady + x), 2);     // one warp of each group
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpQK && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    if (warp == kWarpS) {
        tmem_alloc(smem_u32(tmem_base_ptr), 512);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_ptr;
    auto tS = [&](int b) -> uint32_t { return tmem + 128u * (uint32_t)b; };   // b = step % 3; P aliases it
    const uint32_t tO = tmem + 384u;

    if (warp == kWarpList) {
        // ------------------------------------------------------------ list builder
        int n = 0;
        const long long per_group = (long long)p.nb * p.g;
        while (true) {
            long long u = 0;
            if (lane == 0)
                u = next_tile(p.tile_ctr, p.tile_base, p.status);
            u = __shfl_sync(0xffffffffu, u, 0);
            const int lb = n & 1;
            if (n >= 2 && !warp_wait(bar(G::kListEmpty + lb), ((n >> 1) - 1) & 1, wc))
                break;
            if (u < 0 || u >= p.n_units) {
                if (lane == 0) {
                    infos[lb].count = -1;
                    mbar_arrive(bar(G::kListFull + lb));
                }
                break;
            }
            const int group = (int)(u / per_group);            // b * Hkv + kvh
            const int rem = (int)(u % per_group);
            const int i = p.nb - 1 - rem / p.g;
            const int b = group / p.Hkv;
            const int h = (group % p.Hkv) * p.g + rem % p.g;
            const uint8_t *row = p.mask + ((size_t)(b * p.Hq + h) * p.nb + i) * p.nb;
            uint16_t *lst = lists + lb * lstride;
            int count = 0;
            for (int j0 = 0; j0 <= i; j0 += 512) {
                const int jb = j0 + lane * 16;
                uint32_t bits = 0;
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int j = jb + k;
                    if (j <= i && __ldg(row + j))
                        bits |= 1u << k;
                }
                const int c = __popc(bits);
                int incl = c;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off)
                        incl += v;
                }
                int pos = count + incl - c;
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    if (bits & (1u << k))
                        lst[pos++] = (uint16_t)(jb + k);
                count += __shfl_sync(0xffffffffu, incl, 31);
            }
            __syncwarp();
            if (lane == 0) {
                TileInfo &inf = infos[lb];
                inf.count = count;
                inf.b = b;
                inf.h = h;
                inf.i = i;
                inf.diag = (count > 0 && lst[count - 1] == i) ? 1 : 0;
                mbar_arrive(bar(G::kListFull + lb));
            }
            ++n;
        }
    } else if (warp == kWarpQK || warp == kWarpV) {
        // ------------------------------------------------------------ TMA producers
        // One stage per step; stage x of a ring of two holds steps x, x + 2, ...
        // (numbered over the CTA's whole run).  Step n may load once the MMA that
        // read step n - 2 has completed: S(n - 2) (s_full) for K, PV(n - 2)
        // (pv_done) for V, both kept per step % 3.  A TMA instruction holds
        // its issuing thread for a long time and one thread's copies complete
        // roughly one after another, so each box of a pair is issued by its own
        // lane, all in one instruction.
        const bool kprod = warp == kWarpQK;
        const int R = kprod ? G::kNK : G::kNV;
        int n = 0, q_it = 0, pr = 0;
        bool ok = true;
        const int bFull = kprod ? G::kKFull : G::kVFull;
        const int bDone = kprod ? G::kSFull : G::kPVDone;
        const uint32_t sX = kprod ? sK : sV;
        while (ok) {
            const int lb = n & 1;
            if (!warp_wait(bar(G::kListFull + lb), (n >> 1) & 1, wc)) {
                ok = false;
                break;
            }
            const TileInfo inf = infos[lb];
            if (inf.count < 0)
                break;
            const uint16_t *lst = lists + lb * lstride;
            const int zkv = inf.b * p.Hkv + inf.h / p.g;
            if (inf.count > 0) {
                if (kprod) {
                    const int qb = q_it % G::kQBufs;
                    if (q_it >= G::kQBufs && !warp_wait(bar(G::kQEmpty + qb), (uint32_t)((q_it / G::kQBufs - 1) & 1), wc)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0)
                        mbar_arrive_expect_tx(bar(G::kQFull + qb), (uint32_t)G::kQBytes);
                    __syncwarp();
                    if (lane < G::kPanels)
                        tma_load_3d(sQ + qb * G::kQBytes + lane * 8192, &tmQ, bar(G::kQFull + qb), lane * 64,
                                    inf.i * 64, inf.b * p.Hq + inf.h);
                    ++q_it;
                }
                const int npairs = (inf.count + 1) >> 1;
                for (int e2 = 0; e2 < npairs; ++e2, ++pr) {
                    const int st = pr % R;
                    if (pr >= R && !warp_wait(bar(bDone + (pr - R) % 3), (uint32_t)(((pr - R) / 3) & 1), wc)) {
                        ok = false;
                        break;
                    }
                    const int nblk = min(2, inf.count - 2 * e2);
                    if (lane == 0)
                        mbar_arrive_expect_tx(bar(bFull + st), (uint32_t)(nblk * G::kBlkBytes));
                    __syncwarp();
                    if (kprod) {
                        // [panel][128 keys]: block c fills rows 64c..64c+63 of every panel.
                        if (lane < nblk * G::kPanels) {
                            const int c = lane / G::kPanels, pn = lane % G::kPanels;
                            tma_load_3d(sX + st * G::kPair + pn * 16384 + c * 8192, &tmK, bar(bFull + st), pn * 64,
                                        lst[2 * e2 + c] * 64, zkv);
                        }
                    } else if (lane < nblk) {
                        // [block][panel][64 keys]: one 4-D box per block.
                        tma_load_4d(sX + st * G::kPair + lane * G::kBlkBytes, &tmV, bar(bFull + st), 0,
                                    lst[2 * e2 + lane] * 64, 0, zkv);
                    }
                }
                if (!ok)
                    break;
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(G::kListEmpty + lb));
            ++n;
        }
        if (!ok && lane == 0) {
            // Drain the copies this warp issued before the CTA exits.
            for (int st = 0; st < R; ++st) {
                int last = pr - 1;
                while (last >= 0 && last % R != st)
                    --last;
                if (last >= 0)
                    mbar_drain(bar(bFull + st), (uint32_t)((last / R) & 1), kDrain);
            }
            if (kprod) {
                for (int qb = 0; qb < G::kQBufs; ++qb) {
                    int last = q_it - 1;
                    while (last >= 0 && last % G::kQBufs != qb)
                        --last;
                    if (last >= 0)
                        mbar_drain(bar(G::kQFull + qb), (uint32_t)((last / G::kQBufs) & 1), kDrain);
                }
            }
        }
    } else if (warp == kWarpS) {
        // ------------------------------------------------------------ S issuer
        if (lane == 0) {
            constexpr uint32_t idS2 = idesc_bf16(64, 128, 0);
            constexpr uint32_t idS1 = idesc_bf16(64, 64, 0);
            // Descriptors advance by (byte offset >> 4) in their start-address field.
            const uint64_t dq0 = smem_desc_sw128(sQ, 16, 1024);
            const uint64_t dk0 = smem_desc_sw128(sK, 16, 1024);
            int n = 0, q_it = 0, g = 0, pr = 0;
            bool ok = true, issued = false;
            while (ok) {
                const int lb = n & 1;
                if (!mbar_wait(bar(G::kListFull + lb), (n >> 1) & 1, wc)) {
                    ok = false;
                    break;
                }
                const int count = infos[lb].count;
                mbar_arrive(bar(G::kListEmpty + lb));
                ++n;
                if (count < 0)
                    break;
                if (count == 0)
                    continue;
                const int qb = q_it % G::kQBufs;
                if (!mbar_wait(bar(G::kQFull + qb), (uint32_t)((q_it / G::kQBufs) & 1), wc)) {
                    ok = false;
                    break;
                }
                const uint64_t dq = dq0 + (uint64_t)((qb * G::kQBytes) >> 4);
                const int steps = (count + 1) >> 1;
                for (int s = 0; s < steps; ++s, ++g, ++pr) {
                    const int st = pr % G::kNK;
                    // K of this step landed; S buffer g % 3 free: PV(g - 3) has read the P
                    // written over it (and so the softmax has read S(g - 3)).
                    if (!mbar_wait(bar(G::kKFull + st), (uint32_t)((pr / G::kNK) & 1), wc) ||
                        (g >= 3 && !mbar_wait(bar(G::kPVDone + g % 3), (uint32_t)(((g - 3) / 3) & 1), wc))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t id = (2 * s + 1 < count) ? idS2 : idS1;
                    const uint64_t dk = dk0 + (uint64_t)((st * G::kPair) >> 4);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t qo = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
                        const uint32_t ko = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
                        mma_ss(tS(g % 3), dq + qo, dk + ko, id, kk > 0 ? 1u : 0u);
                    }
                    issued = true;
                    tc_commit(bar(G::kSFull + g % 3));
                    if (s == steps - 1)
                        tc_commit(bar(G::kQEmpty + qb));
                }
                if (!ok)
                    break;
                ++q_it;
            }
            if (issued) {
                tc_commit(bar(G::kDrain + 0));
                mbar_drain(bar(G::kDrain + 0), 0, kDrain);
            }
        }
    } else if (warp == kWarpPV) {
        // ------------------------------------------------------------ PV issuer
        if (lane == 0) {
            constexpr uint32_t idPV = idesc_bf16(64, D, 1);
            const uint64_t dv0 = smem_desc_sw128(sV, 8192, 1024);
            int n = 0, o_it = 0, g = 0, pr = 0;
            bool ok = true, issued = false;
            while (ok) {
                const int lb = n & 1;
                if (!mbar_wait(bar(G::kListFull + lb), (n >> 1) & 1, wc)) {
                    ok = false;
                    break;
                }
                const int count = infos[lb].count;
                mbar_arrive(bar(G::kListEmpty + lb));
                ++n;
                if (count < 0)
                    break;
                if (count == 0)
                    continue;
                const int steps = (count + 1) >> 1;
                for (int s = 0; s < steps; ++s, ++g, ++pr) {
                    const int st = pr % G::kNV;
                    // The first PV of a tile overwrites O: the previous tile's O must
                    // have been read out (o_free).
                    if (!mbar_wait(bar(G::kPFull + g % 3), (uint32_t)((g / 3) & 1), wc) ||
                        !mbar_wait(bar(G::kVFull + st), (uint32_t)((pr / G::kNV) & 1), wc) ||
                        (s == 0 && o_it >= 1 &&
                         !mbar_wait(bar(G::kOFree + ((o_it - 1) & 1)), (uint32_t)(((o_it - 1) >> 1) & 1), wc))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t dv = dv0 + (uint64_t)((st * G::kPair) >> 4);
                    const uint32_t tp = tS(g % 3);
                    // V stage [block][panel][64 keys]: 16 keys per K step, LBO = next d panel.
                    auto chain = [&](auto nk) {
#pragma unroll
                        for (int kk = 0; kk < decltype(nk)::value; ++kk) {
                            const uint32_t vo = ((kk >> 2) * G::kBlkBytes + (kk & 3) * 2048) >> 4;
                            mma_ts(tO, tp + 8u * kk, dv + vo, idPV, (s == 0 && kk == 0) ? 0u : 1u);
                        }
                    };
                    if (2 * s + 1 < count)
                        chain(std::integral_constant<int, 8>{});
                    else
                        chain(std::integral_constant<int, 4>{});
                    issued = true;
                    tc_commit(bar(G::kPVDone + g % 3));
                    if (s == steps - 1)
                        tc_commit(bar(G::kOFull + (o_it & 1)));
                }
                if (!ok)
                    break;
                ++o_it;
            }
            if (issued) {
                tc_commit(bar(G::kDrain + 1));
                mbar_drain(bar(G::kDrain + 1), 0, kDrain);
            }
        }
    } else if (warp < 2 * kGroupWarps) {
        // ------------------------------------------------------------ softmax + epilogue
        const int grp = warp >> 2;               // steps of parity grp are this group's
        const int qt = warp & 3;                 // TMEM lane quarter: rows 16 qt .. 16 qt + 15
        const int r = qt * 16 + (lane & 15);     // query row of the tile
        const int c = lane >> 4;                 // key block of the step this thread holds; half of d
        const uint32_t lane_off = (uint32_t)(qt * 32) << 16;
        float *mrow = reinterpret_cast<float *>(smem + G::kOffM);      // [step % 2][row]
        float *lrow = reinterpret_cast<float *>(smem + G::kOffL);      // [tile % 2][group][l, m][row]
        const float sl2 = p.scale_log2;
        int n = 0, o_it = 0, g = 0;
        bool ok = true;
        // This group's row sum of a tile (both threads of the row), against the
        // running max m_used of its latest step, handed to the epilogue through
        // l_ready.
        auto publish_l = [&](int slot, float l, float m_used) {
            float *dst = lrow + (slot * 2 + grp) * 2 * 64;
            l += __shfl_xor_sync(0xffffffffu, l, 16);   // the row's two threads (key blocks 0 and 1)
            if (lane < 16) {
                dst[r] = l;
                dst[64 + r] = m_used;
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(G::kLReady + slot * 4 + qt));
        };
        // A finished tile whose O this group reads out (it takes the next step).
        bool pend = false;
        int pb = 0, ph = 0, pi = 0, po_it = 0, pg = 0;
        float pm = 0.f;
        // O -> bf16 -> global (and LSE) for the pending tile, then release O.
        auto epilogue = [&]() -> bool {
            const int slot = po_it & 1;
            if (!warp_wait(bar(G::kLReady + slot * 4 + qt), (uint32_t)((po_it >> 1) & 1), wc))
                return false;
            float pl = 0.f;
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const float lx = lrow[(slot * 2 + x) * 2 * 64 + r];
                const float mx = lrow[(slot * 2 + x) * 2 * 64 + 64 + r];
                if (lx > 0.f)
                    pl += lx * ex2_approx(mx - pm);
            }
            if (!warp_wait(bar(G::kOFull + (po_it & 1)), (uint32_t)((po_it >> 1) & 1), wc))
                return false;
            tc_fence_after();
            const bool row_ok = pi * 64 + r < p.S;   // rows past S (ragged last block) are never stored
            const size_t orow = (size_t)(pb * p.Hq + ph) * p.S + (size_t)pi * 64 + r;
            uint4 *dst = reinterpret_cast<uint4 *>(p.o + orow * D + c * (D / 2));
            const float inv_l = pl > 0.f ? 1.0f / pl : 0.f;
            uint32_t ov[D / 2];
            if constexpr (D == 128)
                tmem_ld16x2_64<D / 2>(tO + lane_off, ov);
            else
                tmem_ld16x2_32<D / 2>(tO + lane_off, ov);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(G::kOFree + (po_it & 1)));
            if (row_ok) {
#pragma unroll
                for (int x = 0; x < D / 16; ++x) {
                    uint32_t w[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        w[k] = pack_bf16x2(__uint_as_float(ov[8 * x + 2 * k]) * inv_l,
                                           __uint_as_float(ov[8 * x + 2 * k + 1]) * inv_l);
                    dst[x] = make_uint4(w[0], w[1], w[2], w[3]);
                }
                if (p.lse != nullptr && c == 0)
                    p.lse[orow] = pl > 0.f ? (pm + __log2f(pl)) * 0.69314718055994530942f : -INFINITY;
            }
            pend = false;
            return true;
        };
        while (ok) {
            const int lb = n & 1;
            if (!warp_wait(bar(G::kListFull + lb), (n >> 1) & 1, wc)) {
                ok = false;
                break;
            }
            const TileInfo inf = infos[lb];
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(G::kListEmpty + lb));
            ++n;
            if (inf.count < 0)
                break;
            const int count = inf.count;
            if (count == 0) {
                // No selected block: O = 0, LSE = -inf (written by group 0).
                if (grp == 0 && inf.i * 64 + r < p.S) {
                    const size_t orow = (size_t)(inf.b * p.Hq + inf.h) * p.S + (size_t)inf.i * 64 + r;
                    uint4 *dst = reinterpret_cast<uint4 *>(p.o + orow * D + c * (D / 2));
#pragma unroll
                    for (int x = 0; x < D / 16; ++x)
                        dst[x] = make_uint4(0u, 0u, 0u, 0u);
                    if (p.lse != nullptr && c == 0)
                        p.lse[orow] = -INFINITY;
                }
                continue;
            }
            const int diag = inf.diag;
            const int steps = (count + 1) >> 1;
            const int g0 = g;
            float l = 0.f, m_used = -INFINITY;
            // One step (global number g, step s of the tile): this thread's 64 scores
            // -> row max -> running max (handed on) -> exponentials -> P.  The last
            // step of a tile (absent second block, diagonal block) is a separate
            // instantiation so the other steps carry no masking code.
            auto step = [&](auto last_c, int s) -> bool {
                constexpr bool kLast = decltype(last_c)::value;
                const int b = g % 3;
                if (!warp_wait(bar(G::kSFull + b), (uint32_t)((g / 3) & 1), wc))
                    return false;
                tc_fence_after();
                uint32_t v[64];
                tmem_ld16x2_64<64>(tS(b) + lane_off, v);
                tmem_wait_ld();
                if constexpr (kLast) {
                    // Keys kept: none for an absent block; up to the query row in the
                    // diagonal block (causal); all otherwise.
                    const int e = 2 * s + c;              // list entry of this thread's key block
                    const int lim = e >= count ? 0 : (diag && e == count - 1) ? r + 1 : 64;
#pragma unroll
                    for (int k = 0; k < 64; ++k)
                        v[k] = k < lim ? v[k] : 0xFF800000u;
                }
                float mx8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mx8[k] = __uint_as_float(v[k]);
#pragma unroll
                for (int k = 8; k < 64; ++k)
                    mx8[k & 7] = fmaxf(mx8[k & 7], __uint_as_float(v[k]));
                float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                 fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16)) * sl2;
                // Running max after step g - 1 (the other group's).  At a tile's first
                // step it is the previous tile's final max, kept for that tile's epilogue.
                float m_prev = -INFINITY;
                if (g >= 1) {
                    const int ps = (g - 1) & 1;
                    if (!warp_wait(bar(G::kMReady + ps * 4 + qt), (uint32_t)(((g - 1) >> 1) & 1), wc))
                        return false;
                    const float mp = mrow[ps * 64 + r];
                    if (s == 0)
                        pm = mp;
                    else
                        m_prev = mp;
                }
                const float m_new = mx > m_prev + 8.0f ? mx : m_prev;
                if (lane < 16)
                    mrow[(g & 1) * 64 + r] = m_new;
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar(G::kMReady + (g & 1) * 4 + qt));
                if (m_new != m_used) {
                    l = m_used == -INFINITY ? 0.f : l * ex2_approx(m_used - m_new);
                    m_used = m_new;
                }
                float ls[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t pk[32];
                const float neg_m = -m_new;
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const float p0 = ex2_approx(fmaf(__uint_as_float(v[2 * k]), sl2, neg_m));
                    const float p1 = ex2_approx(fmaf(__uint_as_float(v[2 * k + 1]), sl2, neg_m));
                    ls[k & 3] += p0 + p1;
                    pk[k] = pack_bf16x2(p0, p1);
                }
                l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
                // O holds this tile's PV up to step g - 1 against m_prev: rescale this
                // thread's half of d when the max moved.
                const bool need = s > 0 && m_new != m_prev;
                if (__any_sync(0xffffffffu, need)) {
                    const float alpha = need ? ex2_approx(m_prev - m_new) : 1.0f;
                    if (!warp_wait(bar(G::kPVDone + (g - 1) % 3), (uint32_t)(((g - 1) / 3) & 1), wc))
                        return false;
                    tc_fence_after();
#pragma unroll 1
                    for (int ch = 0; ch < D / 32; ++ch) {
                        uint32_t ov[16];
                        tmem_ld16x2_16<D / 2>(tO + lane_off + ch * 16, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
                        tmem_st16x2_16<D / 2>(tO + lane_off + ch * 16, ov);
                    }
                    tmem_wait_st();
                }
                // P over the first 64 columns of this S buffer: only this warp reads
                // these lanes of it, and its loads have completed.  Keys 2k, 2k + 1
                // of block c go to column 32 c + k.
                tmem_st16x2_32<32>(tS(b) + lane_off, pk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar(G::kPFull + b));
                // The previous tile's O: its last PV finished while this step ran;
                // this tile's first PV waits for it to be read out.
                if (pend && !epilogue())
                    return false;
                return true;
            };
            int s = (g0 & 1) == grp ? 0 : 1;
            if (s >= steps)
                publish_l(o_it & 1, 0.f, -INFINITY);   // a one-step tile of the other group
            for (; s < steps; s += 2) {
                g = g0 + s;
                const bool good = (s + 1 < steps) ? step(std::false_type{}, s) : step(std::true_type{}, s);
                if (!good) {
                    ok = false;
                    break;
                }
                if (s + 2 >= steps)
                    publish_l(o_it & 1, l, m_used);
            }
            if (!ok)
                break;
            g = g0 + steps;
            // The group that takes the next step reads this tile's O out.
            if ((g & 1) == grp) {
                pend = true;
                pb = inf.b;
                ph = inf.h;
                pi = inf.i;
                po_it = o_it;
                pg = g - 1;
            }
            ++o_it;
        }
        if (ok && pend) {
            // No further step: take the pending tile's final max, then read O out.
            const int ps = pg & 1;
            if (warp_wait(bar(G::kMReady + ps * 4 + qt), (uint32_t)((pg >> 1) & 1), wc)) {
                pm = mrow[ps * 64 + r];
                epilogue();
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpS) {
        tc_fence_after();
        tmem_dealloc(*tmem_base_ptr, 512);
    }
}

template <int D>
cudaError_t launch_d(const AttnLaunch &a, cudaStream_t stream)
{
    CUtensorMap tq, tk, tv;
    if (!make_tmap_bhsd(&tq, a.q, a.B * a.Hq, a.S, D) || !make_tmap_bhsd(&tk, a.k, a.B * a.Hkv, a.S, D) ||
        !make_tmap_bhsd_panels(&tv, a.v, a.B * a.Hkv, a.S, D))
        return cudaErrorInvalidValue;
    SParams p{};
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.S = a.S;
    p.nb = a.nb;
    p.g = a.Hq / a.Hkv;
    p.n_units = (long long)a.B * a.Hq * a.nb;
    p.scale_log2 = a.scale_log2;
    p.mask = a.mask;
    p.o = reinterpret_cast<__nv_bfloat16 *>(a.o);
    p.lse = a.lse;
    p.timeout_ns = a.timeout_ns;
    p.status = a.status;
    p.tile_ctr = a.tile_ctr;
    p.tile_base = a.tile_base;
    p.list_stride = Geo<D>::list_stride(a.nb);
    const int smem = Geo<D>::smem_bytes(a.nb);
    if (Geo<D>::smem_used(a.nb) > 227 * 1024)
        return cudaErrorInvalidValue;
    auto kern = sparse_attn_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // One persistent CTA per SM (a kernel that allocates all of TMEM runs one per SM).
    long long grid = p.n_units < sms ? p.n_units : sms;
    if (grid < 1)
        grid = 1;
    kern<<<(unsigned)grid, kThreads, smem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_sparse_attention(const AttnLaunch &a, cudaStream_t stream)
{
    if (a.d == 128)
        return launch_d<128>(a, stream);
    if (a.d == 64)
        return launch_d<64>(a, stream);
    return cudaErrorInvalidValue;
}

} // namespace seer
