// seer_attn.cu — block-sparse causal attention prefill and the Figure-8
// pooled-map pass, written for sm_100a (TMA + tcgen05 + TMEM).
//
// What it computes:
//  * sparse mode ("Learning Intrinsic Sparse Attention in Your LLMs",
//    rebuttal Weakness 5, inference kernel pseudocode): for each query block,
//    an online softmax over the selected key blocks only.
//  * map mode ("SeerAttention: Self-distilled Attention Gating", Figure 8):
//    dense causal attention that also stores the per-row block maxima r_ij
//    and afterwards turns them into A_ij = colmax(exp(r_ij - m_i) / l_i).
//
// B200 design (differs from the pages' FA-2/Triton kernels on A100):
//  * One tensor-core tile is 128 query rows = two 64-row "halves" that read
//    the same KV head: two query heads of one GQA group at the same query
//    block, or (for the leftover head of an odd group) two adjacent query
//    blocks of one head.  The tile walks the UNION of the halves' active key
//    blocks; a block that only one half selected gets P = 0 for the other
//    half's rows and leaves that half's running max/sum untouched, which is
//    exact.  M = 128 keeps tcgen05.mma at its full per-SM rate.
//  * S = Q K^T (SS MMA, N = 64) and O += P V (TS MMA: P read from TMEM) with
//    fp32 accumulators in TMEM: S double-buffered (2 x 64 columns, P aliased
//    into the first 32 columns of its S buffer), O in 128 columns.
//  * One CTA per SM (a kernel that allocates TMEM is granted one CTA per SM)
//    with two independent tile slots.  Per slot: warps 0-3 softmax / rescale /
//    epilogue (thread = row = TMEM lane), warp 4 TMA producer for Q and K,
//    warp 5 MMA issuer, warp 6 builds the per-tile active-block list from the
//    mask (the compaction step, fused so skipped blocks cost no loads and no
//    extra launch), warp 7 TMA producer for V.
//  * Persistent grid; tiles are KV-head major (concurrent tiles share one KV
//    head's K/V in L2), heaviest query blocks first, and each slot takes the
//    next tile from a launch-wide atomic counter when it is ready for one
//    (a static round-robin left the busiest SM with 8-9 % more work than the
//    mean, dense or sparse).
//  * The running max is only moved when it grows by more than 2^8 (log2
//    domain); P = 2^(x - m) then stays <= 256, safe in bf16/fp32, and the O
//    rescale (TMEM load/store) is rare.
//  * Every wait is bounded (seer_ptx.cuh); a wait that runs out raises the
//    status word, the CTA drains its in-flight copies and MMAs, frees TMEM and
//    exits.
#include <cuda_bf16.h>

#include "seer_internal.h"
#include "seer_ptx.cuh"

namespace seer {

namespace {

constexpr int kNStage = 2;            // K/V pipeline depth
constexpr int kPrefetch = 4;          // L2 prefetch distance (key blocks)
constexpr int kRows = 128;            // rows of one tile (two halves of 64)
constexpr uint64_t kDrainNs = 200000000ull;

struct UnitInfo {
    int count, b, h0, i0, h1, i1;
};

struct Unit {
    int b, kvh, h0, i0, h1, i1;
    bool valid;
};

struct KParams {
    int B, Hq, Hkv, S, nb, g, lanes;
    long long n_units;
    float scale_log2;
    const uint8_t *mask;
    __nv_bfloat16 *o;
    float *lse;
    float *A;
    float *rscratch;
    uint64_t timeout_ns;
    int *status;
    int nslots;              // independent tiles in flight per CTA (1 or 2)
    int slot_bytes;          // shared memory per slot
    unsigned long long *tile_ctr;   // next tile of the launch (seeded with tile_base before it)
    unsigned long long tile_base;
};

// Tile order: KV-head major, so the CTAs running at any moment read the K/V
// of one or two KV heads (a few tens of MB: L2-resident).  Inside a KV head,
// level = 0 is the last query block (the longest causal rows) and levels go
// down, so heavy tiles come first.  Within a level, lane < g/2 pairs heads
// (2l, 2l+1) of the group at the same query block; the last lane of an odd
// group pairs the leftover head's blocks (i, i-1) on even levels and is empty
// on odd levels.
__device__ __forceinline__ Unit decode_unit(const KParams &p, long long u)
{
    const long long per_group = (long long)p.nb * p.lanes;
    const int group = (int)(u / per_group);          // b * Hkv + kvh
    const int rem = (int)(u % per_group);
    const int level = rem / p.lanes;
    const int lane = rem % p.lanes;
    const int kvh = group % p.Hkv;
    const int b = group / p.Hkv;
    const int i = p.nb - 1 - level;
    Unit r;
    r.b = b;
    r.kvh = kvh;
    r.valid = true;
    if (lane < p.g / 2) {
        r.h0 = kvh * p.g + 2 * lane;
        r.h1 = r.h0 + 1;
        r.i0 = r.i1 = i;
    } else {
        r.h0 = r.h1 = kvh * p.g + p.g - 1;
        r.i0 = i;
        r.i1 = i - 1;
        if (level & 1)
            r.valid = false;
        if (r.i1 < 0)
            r.h1 = -1;
    }
    return r;
}

template <int D>
struct Smem {
    static constexpr int kPanels = D / 64;
    static constexpr int kQPanelBytes = kRows * 128;      // 128 rows x 128 B
    static constexpr int kQBytes = kPanels * kQPanelBytes;
    static constexpr int kKVPanelBytes = 64 * 128;        // 64 keys x 128 B
    static constexpr int kKVBytes = kPanels * kKVPanelBytes;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + kNStage * kKVBytes;
    static constexpr int kOffBar = kOffV + kNStage * kKVBytes;
    // barriers (8 B each)
    static constexpr int kBarQFull = 0, kBarQEmpty = 1, kBarKFull = 2, kBarVFull = 2 + kNStage,
                         kBarKEmpty = 2 + 2 * kNStage, kBarVEmpty = 2 + 3 * kNStage, kBarSFull = 2 + 4 * kNStage,
                         kBarPFull = kBarSFull + 2, kBarODone = kBarPFull + 2, kBarOFree = kBarODone + 2,
                         kBarListFull = kBarOFree + 1, kBarListEmpty = kBarListFull + 2,
                         kBarDrain = kBarListEmpty + 2, kNumBars = kBarDrain + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;   // tmem base, abort flag
    static constexpr int kOffInfo = (kOffMisc + 16 + 15) / 16 * 16;
    static constexpr int kOffRed = kOffInfo + 2 * (int)sizeof(UnitInfo) + 16;
    static constexpr int kOffList = (kOffRed + 4 * 32 * 4 + 15) / 16 * 16;
    static constexpr int kBaseBytes = kOffList;
    // One slot: Q, K/V ring, barriers, unit info and two list buffers; slots
    // start on 1024-B boundaries (the 128-B swizzle pattern repeats every 1 KB).
    static int slot_bytes(int nb) { return (kBaseBytes + 2 * ((nb * 2 + 15) / 16 * 16) + 1023) / 1024 * 1024; }
    static int total_bytes(int nb, int nslots) { return nslots * slot_bytes(nb) + 1024; }
};

__device__ __forceinline__ float warp_max_transpose32(float (&v)[32], int lane)
{
    // After this, lane L holds max over lanes of v[L].
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) {
        const bool upper = (lane & k) != 0;
#pragma unroll
        for (int i = 0; i < k; ++i) {
            const float send = upper ? v[i] : v[i + k];
            const float keep = upper ? v[i + k] : v[i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, k);
            v[i] = fmaxf(keep, recv);
        }
    }
    return v[0];
}

// All 32 lanes poll; the warp proceeds only if every lane saw the phase, so a
// timeout can never split a warp in front of a .sync.aligned instruction.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitCtx &w)
{
    const bool r = mbar_wait(bar, parity, w);
    return __all_sync(0xffffffffu, r);
}

template <int D, bool MAP>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const KParams p)
{
    using L = Smem<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // Align the dynamic window to 1024 B.
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Two slots per CTA (one CTA per SM: TMEM allocation pins occupancy to 1).
    // Each slot is an independent tile pipeline: warps 8s+0..3 softmax (TMEM
    // lane quarters 0..3), 8s+4 Q/K producer, 8s+5 MMA issuer, 8s+6 list
    // builder, 8s+7 V producer.  Slot s owns TMEM columns [256 s, 256 s + 256).
    const int slot = warp >> 3;
    const int wl = warp & 7;
    uint8_t *ssm = smem + slot * p.slot_bytes;
    const uint32_t sbase = smem_u32(ssm);
    const uint32_t sQ = sbase + L::kOffQ;
    const uint32_t sK = sbase + L::kOffK;
    const uint32_t sV = sbase + L::kOffV;
    const uint32_t sBar = sbase + L::kOffBar;
    auto bar = [&](int idx) -> uint32_t { return sBar + 8u * idx; };
    uint32_t *tmem_base_ptr = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
    UnitInfo *infos = reinterpret_cast<UnitInfo *>(ssm + L::kOffInfo);
    const int list_stride = (p.nb * 2 + 15) / 16 * 8;   // uint16 entries per buffer
    uint16_t *lists = reinterpret_cast<uint16_t *>(ssm + L::kOffList);
    const WaitCtx wc{abort_flag, p.timeout_ns, p.status};

    if (threadIdx.x == 0) {
        for (int sl = 0; sl < p.nslots; ++sl) {
            const uint32_t sb0 = smem_u32(smem + sl * p.slot_bytes) + L::kOffBar;
            auto bi = [&](int idx) -> uint32_t { return sb0 + 8u * idx; };
            mbar_init(bi(L::kBarQFull), 1);
            mbar_init(bi(L::kBarQEmpty), 1);
            for (int s = 0; s < kNStage; ++s) {
                mbar_init(bi(L::kBarKFull + s), 1);
                mbar_init(bi(L::kBarVFull + s), 1);
                mbar_init(bi(L::kBarKEmpty + s), 1);
                mbar_init(bi(L::kBarVEmpty + s), 1);
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(bi(L::kBarSFull + b), 1);
                mbar_init(bi(L::kBarPFull + b), kRows);
                mbar_init(bi(L::kBarListFull + b), 1);
                mbar_init(bi(L::kBarListEmpty + b), 7);
            }
            mbar_init(bi(L::kBarODone + 0), 1);
            mbar_init(bi(L::kBarODone + 1), 1);
            mbar_init(bi(L::kBarOFree), kRows);
            mbar_init(bi(L::kBarDrain), 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 4 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(tmem_base_ptr), 512);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_ptr + 256u * (uint32_t)slot;
    auto tS = [&](int b) -> uint32_t { return tmem + 64u * (uint32_t)b; };
    const uint32_t tO = tmem + 128u;

    // Virtual CTA: this slot's index (its Figure-8 scratch region).
    const long long vcta = (long long)blockIdx.x * p.nslots + slot;
    const bool slot_on = slot < p.nslots;

    if (!slot_on) {
        // idle slot (the tiles' shared memory did not fit twice)
    } else if (wl == 6) {
        // ------------------------------------------------------------ list builder
        // Tiles are taken from a launch-wide counter in the persistent order
        // (dynamic scheduling: a slot that finishes early takes the next tile);
        // the builder publishes each tile, then a count of -1 that ends the
        // slot's other roles.
        int n = 0;
        while (true) {
            long long u = 0;
            if (lane == 0)
                u = next_tile(p.tile_ctr, p.tile_base, p.status);
            u = __shfl_sync(0xffffffffu, u, 0);
            const bool end = u < 0 || u >= p.n_units;
            Unit un{};
            if (!end) {
                un = decode_unit(p, u);
                if (!un.valid)
                    continue;
            }
            const int lb = n & 1;
            const int fill = n >> 1;
            if (fill >= 1 && !warp_wait(bar(L::kBarListEmpty + lb), (fill - 1) & 1, wc))
                break;
            if (end) {
                if (lane == 0) {
                    infos[lb].count = -1;
                    mbar_arrive(bar(L::kBarListFull + lb));
                }
                break;
            }
            uint16_t *lst = lists + lb * list_stride;
            int count = 0;
            if (MAP) {
                count = un.i0 + 1;
                for (int j = lane; j < count; j += 32) {
                    const int a1 = (un.h1 >= 0 && j <= un.i1) ? 1 : 0;
                    lst[j] = (uint16_t)(j | (1 << 14) | (a1 << 15));
                }
            } else {
                const uint8_t *row0 = p.mask + ((size_t)(un.b * p.Hq + un.h0) * p.nb + un.i0) * p.nb;
                const uint8_t *row1 =
                    un.h1 >= 0 ? p.mask + ((size_t)(un.b * p.Hq + un.h1) * p.nb + un.i1) * p.nb : nullptr;
                for (int j0 = 0; j0 <= un.i0; j0 += 512) {
                    const int jb = j0 + lane * 16;
                    uint32_t bits0 = 0, bits1 = 0;
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const int j = jb + k;
                        if (j <= un.i0 && __ldg(row0 + j))
                            bits0 |= 1u << k;
                        if (row1 != nullptr && j <= un.i1 && __ldg(row1 + j))
                            bits1 |= 1u << k;
                    }
                    const uint32_t act = bits0 | bits1;
                    const int c = __popc(act);
                    int incl = c;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const int v = __shfl_up_sync(0xffffffffu, incl, off);
                        if (lane >= off)
                            incl += v;
                    }
                    int pos = count + incl - c;
                    const int total = __shfl_sync(0xffffffffu, incl, 31);
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        if (act & (1u << k)) {
                            lst[pos++] = (uint16_t)((jb + k) | (((bits0 >> k) & 1u) << 14) |
                                                    (((bits1 >> k) & 1u) << 15));
                        }
                    }
                    count += total;
                }
            }
            if (lane == 0) {
                UnitInfo &inf = infos[lb];
                inf.count = count;
                inf.b = un.b;
                inf.h0 = un.h0;
                inf.i0 = un.i0;
                inf.h1 = un.h1;
                inf.i1 = un.i1;
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(L::kBarListFull + lb));
            ++n;
        }
    } else if (wl == 4 || wl == 7) {
        // ------------------------------------------------------------ TMA producers
        // Warp 4 loads Q and K, warp 7 loads V: a V stage that waits for a late
        // PV must not hold back the next K tile (S needs K long before PV needs V).
        const bool kprod = wl == 4;
        if (lane == 0) {
            int n = 0, q_it = 0;
            long long kv_it = 0;
            bool ok = true;
            const CUtensorMap *tm = kprod ? &tmK : &tmV;
            const uint32_t sX = kprod ? sK : sV;
            const int bFull = kprod ? L::kBarKFull : L::kBarVFull;
            const int bEmpty = kprod ? L::kBarKEmpty : L::kBarVEmpty;
            while (ok) {
                const int lb = n & 1;
                if (!mbar_wait(bar(L::kBarListFull + lb), (n >> 1) & 1, wc)) {
                    ok = false;
                    break;
                }
                const UnitInfo inf = infos[lb];
                if (inf.count < 0)
                    break;
                const uint16_t *lst = lists + lb * list_stride;
                if (inf.count > 0) {
                    if (kprod) {
                        if (q_it >= 1 && !mbar_wait(bar(L::kBarQEmpty), (q_it - 1) & 1, wc)) {
                            ok = false;
                            break;
                        }
                        const int halves = inf.h1 >= 0 ? 2 : 1;
                        mbar_arrive_expect_tx(bar(L::kBarQFull), (uint32_t)(halves * 64 * D * 2));
                        for (int hf = 0; hf < halves; ++hf) {
                            const int h = hf ? inf.h1 : inf.h0;
                            const int i = hf ? inf.i1 : inf.i0;
#pragma unroll
                            for (int pn = 0; pn < L::kPanels; ++pn)
                                tma_load_3d(sQ + pn * L::kQPanelBytes + hf * 8192, &tmQ, bar(L::kBarQFull), pn * 64,
                                            i * 64, inf.b * p.Hq + h);
                        }
                        ++q_it;
                    }
                    const int zkv = inf.b * p.Hkv + inf.h0 / p.g;
                    for (int t = 0; t < inf.count; ++t) {
                        const int j = lst[t] & 0x3FFF;
                        const int s = (int)(kv_it % kNStage);
                        const long long use = kv_it / kNStage;
                        if (use >= 1 && !mbar_wait(bar(bEmpty + s), (uint32_t)((use - 1) & 1), wc)) {
                            ok = false;
                            break;
                        }
                        // One box: 64 keys x all d/64 panels (panel-major, 8 KB per panel).
                        mbar_arrive_expect_tx(bar(bFull + s), (uint32_t)(64 * D * 2));
                        tma_load_4d(sX + s * L::kKVBytes, tm, bar(bFull + s), 0, j * 64, 0, zkv);
                        // Warm L2 with the block kPrefetch positions ahead.
                        if (t + kPrefetch < inf.count) {
                            const int jp = lst[t + kPrefetch] & 0x3FFF;
                            tma_prefetch_4d(tm, 0, jp * 64, 0, zkv);
                        }
                        ++kv_it;
                    }
                    if (!ok)
                        break;
                }
                mbar_arrive(bar(L::kBarListEmpty + lb));
                ++n;
            }
            if (!ok) {
                // Drain the loads this thread issued before leaving.
                for (int s = 0; s < kNStage; ++s) {
                    if (kv_it > s) {
                        const long long last = ((kv_it - 1 - s) / kNStage) * kNStage + s;
                        mbar_drain(bar(bFull + s), (uint32_t)((last / kNStage) & 1), kDrainNs);
                    }
                }
                if (kprod && q_it > 0)
                    mbar_drain(bar(L::kBarQFull), (q_it - 1) & 1, kDrainNs);
            }
        }
    } else if (wl == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 64, 0);
            constexpr uint32_t idPV = idesc_bf16(128, D, 1);
            int n = 0, q_it = 0, o_units = 0;
            long long kv_base = 0, sb = 0;
            bool ok = true;
            bool issued = false;
            while (ok) {
                const int lb = n & 1;
                if (!mbar_wait(bar(L::kBarListFull + lb), (n >> 1) & 1, wc)) {
                    ok = false;
                    break;
                }
                const int count = infos[lb].count;
                if (count < 0)
                    break;
                if (count > 0) {
                    if (!mbar_wait(bar(L::kBarQFull), q_it & 1, wc)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int t = 0; t <= count && ok; ++t) {
                        if (t < count) {
                            const long long it = kv_base + t;
                            const int s = (int)(it % kNStage);
                            if (!mbar_wait(bar(L::kBarKFull + s), (uint32_t)((it / kNStage) & 1), wc)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const int b = (int)((sb + t) & 1);
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint64_t da = smem_desc_sw128(sQ + (kk >> 2) * L::kQPanelBytes + (kk & 3) * 32,
                                                                    16, 1024);
                                const uint64_t db = smem_desc_sw128(
                                    sK + s * L::kKVBytes + (kk >> 2) * L::kKVPanelBytes + (kk & 3) * 32, 16, 1024);
                                mma_ss(tS(b), da, db, idS, kk > 0 ? 1u : 0u);
                            }
                            issued = true;
                            tc_commit(bar(L::kBarSFull + b));
                            tc_commit(bar(L::kBarKEmpty + s));
                            if (t == count - 1)
                                tc_commit(bar(L::kBarQEmpty));
                        }
                        if (t >= 1) {
                            const int tp = t - 1;
                            const long long it = kv_base + tp;
                            const int s = (int)(it % kNStage);
                            const int b = (int)((sb + tp) & 1);
                            if (!mbar_wait(bar(L::kBarPFull + b), (uint32_t)(((sb + tp) >> 1) & 1), wc) ||
                                !mbar_wait(bar(L::kBarVFull + s), (uint32_t)((it / kNStage) & 1), wc)) {
                                ok = false;
                                break;
                            }
                            if (tp == 0 && o_units >= 1 &&
                                !mbar_wait(bar(L::kBarOFree), (uint32_t)((o_units - 1) & 1), wc)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                // V tile is MN-major: 16 keys x D; LBO = next 64 columns (panel), SBO = 8 keys.
                                const uint64_t dv =
                                    smem_desc_sw128(sV + s * L::kKVBytes + kk * 16 * 128, L::kKVPanelBytes, 1024);
                                mma_ts(tO, tS(b) + kk * 8, dv, idPV, (tp > 0 || kk > 0) ? 1u : 0u);
                            }
                            tc_commit(bar(L::kBarVEmpty + s));
                            tc_commit(bar(L::kBarODone + (int)(it & 1)));
                        }
                    }
                    if (!ok)
                        break;
                    kv_base += count;
                    sb += count;
                    ++q_it;
                    ++o_units;
                }
                mbar_arrive(bar(L::kBarListEmpty + lb));
                ++n;
            }
            if (issued) {
                // Wait for every MMA this thread issued before TMEM is freed.
                tc_commit(bar(L::kBarDrain));
                mbar_drain(bar(L::kBarDrain), 0, kDrainNs);
            }
        }
    } else if (wl < 4) {
        // ------------------------------------------------------------ softmax / epilogue
        const int row = wl * 32 + lane;       // 0..127 == TMEM lane
        const int half = row >> 6;
        const int r_in = row & 63;
        const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
        int n = 0;
        long long sb = 0, pv_total = 0;
        // PV number n (counted over the CTA's lifetime) arrives on o_done[n & 1].
        // A parity wait only separates a phase from the one just before it;
        // whenever a softmax warp waits for PV n, PV n-2 is already known to be
        // complete (the S tile it just read was committed after PV n-2) and PV
        // n+2 cannot start without this warp, so barrier n & 1 is exactly at
        // phase n >> 1 or one past it.
        auto wait_pv = [&](long long n_pv) -> bool {
            return warp_wait(bar(L::kBarODone + (int)(n_pv & 1)), (uint32_t)((n_pv >> 1) & 1), wc);
        };
        float *rs = MAP ? p.rscratch + (size_t)vcta * p.nb * kRows : nullptr;
        bool ok = true;
        while (ok) {
            const int lb = n & 1;
            if (!warp_wait(bar(L::kBarListFull + lb), (n >> 1) & 1, wc)) {
                ok = false;
                break;
            }
            const UnitInfo inf = infos[lb];
            if (inf.count < 0)
                break;
            const uint16_t *lst = lists + lb * list_stride;
            const int my_h = half ? inf.h1 : inf.h0;
            const int my_i = half ? inf.i1 : inf.i0;
            const bool present = my_h >= 0;
            float m = -INFINITY, l = 0.f;
            for (int t = 0; t < inf.count; ++t) {
                const int b = (int)(sb & 1);
                if (!warp_wait(bar(L::kBarSFull + b), (uint32_t)((sb >> 1) & 1), wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t e = lst[t];
                const int j = (int)(e & 0x3FFF);
                const bool act = present && ((e >> (14 + half)) & 1u);
                if (act) {
                    uint32_t s0[32], s1[32];
                    tmem_ld32(tS(b) + lane_off, s0);
                    tmem_ld32(tS(b) + lane_off + 32, s1);
                    tmem_wait_ld();
                    if (j == my_i) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            if (c > r_in)
                                s0[c] = 0xFF800000u;   // -inf: key after the query (causal)
                            if (c + 32 > r_in)
                                s1[c] = 0xFF800000u;
                        }
                    }
                    float rmax = __uint_as_float(s0[0]);
#pragma unroll
                    for (int c = 1; c < 32; ++c)
                        rmax = fmaxf(rmax, __uint_as_float(s0[c]));
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        rmax = fmaxf(rmax, __uint_as_float(s1[c]));
                    rmax *= p.scale_log2;
                    if (MAP)
                        rs[(size_t)t * kRows + row] = rmax;
                    const bool grow = rmax > m + 8.0f;
                    const float m_new = grow ? rmax : m;
                    // Rescale O only when some row of this warp moved its max and
                    // already has contributions (m finite).
                    const bool need = grow && (m != -INFINITY);
                    if (__any_sync(0xffffffffu, need)) {
                        const float alpha = need ? ex2_approx(m - m_new) : 1.0f;
                        l *= alpha;
                        if (!wait_pv(pv_total + t - 1)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll 1
                        for (int ch = 0; ch < D / 16; ++ch) {
                            uint32_t ov[16];
                            tmem_ld16(tO + lane_off + ch * 16, ov);
                            tmem_wait_ld();
#pragma unroll
                            for (int c = 0; c < 16; ++c)
                                ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
                            tmem_st16(tO + lane_off + ch * 16, ov);
                        }
                    }
                    m = m_new;
                    const float neg_m = -m;
                    float lsum = 0.f;
                    {
                        uint32_t pk[16];
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const float p0 = ex2_approx(fmaf(__uint_as_float(s0[2 * c]), p.scale_log2, neg_m));
                            const float p1 = ex2_approx(fmaf(__uint_as_float(s0[2 * c + 1]), p.scale_log2, neg_m));
                            lsum += p0 + p1;
                            pk[c] = pack_bf16x2(p0, p1);
                        }
                        tmem_st16(tS(b) + lane_off, pk);
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const float p0 = ex2_approx(fmaf(__uint_as_float(s1[2 * c]), p.scale_log2, neg_m));
                            const float p1 = ex2_approx(fmaf(__uint_as_float(s1[2 * c + 1]), p.scale_log2, neg_m));
                            lsum += p0 + p1;
                            pk[c] = pack_bf16x2(p0, p1);
                        }
                        tmem_st16(tS(b) + lane_off + 16, pk);
                    }
                    l += lsum;
                } else {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        pk[c] = 0u;
                    tmem_st16(tS(b) + lane_off, pk);
                    tmem_st16(tS(b) + lane_off + 16, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(L::kBarPFull + b));
                ++sb;
            }
            if (!ok)
                break;
            // -------------------------------------------------- epilogue
            if (inf.count > 0) {
                if (!wait_pv(pv_total + inf.count - 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            // A ragged last block has rows past S: they were computed from the
            // zero rows TMA fills in, and are neither stored nor pooled (the
            // TMEM reads below stay warp-uniform; only the stores are per row).
            const bool row_ok = present && my_i * 64 + r_in < p.S;
            if (present) {
                const size_t orow = ((size_t)(inf.b * p.Hq + my_h) * p.S + (size_t)my_i * 64 + r_in);
                uint4 *dst = reinterpret_cast<uint4 *>(p.o + orow * D);
                const bool has = inf.count > 0 && l > 0.f;
                const float inv_l = has ? 1.0f / l : 0.f;
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch) {
                    uint32_t ov[32];
                    if (inf.count > 0) {
                        tmem_ld32(tO + lane_off + ch * 32, ov);
                        tmem_wait_ld();
                    }
                    uint32_t pkd[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float a0 = has ? __uint_as_float(ov[2 * c]) * inv_l : 0.f;
                        const float a1 = has ? __uint_as_float(ov[2 * c + 1]) * inv_l : 0.f;
                        pkd[c] = pack_bf16x2(a0, a1);
                    }
                    if (row_ok) {
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[ch * 4 + v4] =
                                make_uint4(pkd[4 * v4], pkd[4 * v4 + 1], pkd[4 * v4 + 2], pkd[4 * v4 + 3]);
                    }
                }
                if (p.lse != nullptr && row_ok)
                    p.lse[orow] = has ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
            }
            if (inf.count > 0) {
                tc_fence_before();
                mbar_arrive(bar(L::kBarOFree));
            }
            if (MAP) {
                // Figure 8 second pass: a_ij = 2^(r_ij - m) / l, A_ij = max over the 64 rows.
                const float inv_l = (row_ok && l > 0.f) ? 1.0f / l : 0.f;
                float *Arow = present ? p.A + ((size_t)(inf.b * p.Hq + my_h) * p.nb + my_i) * p.nb : nullptr;
                for (int t0 = 0; t0 < inf.count; t0 += 32) {
                    float vals[32];
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const int t = t0 + k;
                        vals[k] = (row_ok && t < inf.count && t <= my_i)
                                      ? ex2_approx(rs[(size_t)t * kRows + row] - m) * inv_l
                                      : 0.f;
                    }
                    // Lane L now holds the max over this warp's 32 rows for block t0 + L;
                    // the two warps of a half meet in global memory (A was zeroed).
                    const float wmax = warp_max_transpose32(vals, lane);
                    const int jj = t0 + lane;
                    if (present && jj <= my_i && jj < inf.count)
                        atomicMax(reinterpret_cast<int *>(Arow + jj), __float_as_int(wmax));
                }
            }
            pv_total += inf.count;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(L::kBarListEmpty + lb));
            ++n;
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(*tmem_base_ptr, 512);
    }
}

template <int D, bool MAP>
cudaError_t launch_t(const AttnLaunch &a, cudaStream_t stream)
{
    CUtensorMap tq, tk, tv;
    if (!make_tmap_bhsd(&tq, a.q, a.B * a.Hq, a.S, D) || !make_tmap_bhsd_panels(&tk, a.k, a.B * a.Hkv, a.S, D) ||
        !make_tmap_bhsd_panels(&tv, a.v, a.B * a.Hkv, a.S, D))
        return cudaErrorInvalidValue;
    KParams p;
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.S = a.S;
    p.nb = a.nb;
    p.g = a.Hq / a.Hkv;
    p.lanes = (p.g + 1) / 2;
    p.n_units = (long long)a.nb * a.B * a.Hkv * p.lanes;
    p.scale_log2 = a.scale_log2;
    p.mask = a.mask;
    p.o = reinterpret_cast<__nv_bfloat16 *>(a.o);
    p.lse = a.lse;
    p.A = a.A;
    p.rscratch = a.rscratch;
    p.timeout_ns = a.timeout_ns;
    p.status = a.status;
    p.tile_ctr = a.tile_ctr;
    p.tile_base = a.tile_base;
    // Two tile slots per CTA when their shared memory fits (227 KB per CTA).
    p.nslots = Smem<D>::total_bytes(a.nb, 2) <= 227 * 1024 ? 2 : 1;
    p.slot_bytes = Smem<D>::slot_bytes(a.nb);
    const int smem = Smem<D>::total_bytes(a.nb, p.nslots);
    auto kern = attn_kernel<D, MAP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // One persistent CTA per SM (kernels that allocate TMEM run one CTA per SM).
    const long long vctas = attn_grid_size(a.B, a.Hq, a.Hkv, a.nb);
    long long grid = (vctas + p.nslots - 1) / p.nslots;
    if (grid > sms)
        grid = sms;
    if (grid < 1)
        grid = 1;
    kern<<<(unsigned)grid, kAttnThreads, smem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

} // namespace

int attn_grid_size(int B, int Hq, int Hkv, int nb)
{
    static int sms = 0;
    if (sms == 0) {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            sms = v;
        else
            sms = 148;
    }
    const int g = Hq / Hkv;
    const long long units = (long long)nb * B * Hkv * ((g + 1) / 2);
    long long grid = 2LL * sms;
    if (grid > kMaxAttnCtas)
        grid = kMaxAttnCtas;
    if (grid > units)
        grid = units;
    return (int)(grid < 1 ? 1 : grid);
}

cudaError_t launch_attention(const AttnLaunch &a, cudaStream_t stream)
{
    if (!a.map_mode)
        return launch_sparse_attention(a, stream);
    if (a.d == 128)
        return a.map_mode ? launch_t<128, true>(a, stream) : launch_t<128, false>(a, stream);
    if (a.d == 64)
        return a.map_mode ? launch_t<64, true>(a, stream) : launch_t<64, false>(a, stream);
    return cudaErrorInvalidValue;
}

} // namespace seer
