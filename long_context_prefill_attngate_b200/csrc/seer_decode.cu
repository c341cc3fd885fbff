// seer_decode.cu — block-sparse attention of one new token per sequence over
// its KV cache: the decode step of "SeerAttention-R: Sparse Attention
// Adaptation for Long Reasoning" (the gate without query pooling selects KV
// blocks; a sparse decoding kernel reads only those).
//
// o[b,h] = sum over keys c < L in active blocks of softmax(q . k_c * scale) v_c
// for the token at position L - 1 (every cached key is at or before it).
//
// Decode reads each active K/V block once and does 2 x 64 x d flops per block
// with them: it is bound by HBM (and L2, for blocks the heads of a GQA group
// share), so this is a CUDA-core kernel sized for memory parallelism, not a
// tensor-core one:
//  * split-K over the active blocks (flash-decoding): CTA (split s, head bh)
//    takes the active blocks whose rank in the mask row is s mod nsplit, keeps
//    an online softmax and writes (o, m, l) partials; a second kernel merges
//    the splits and normalises.
//  * per block: 128 threads = 64 keys x 2 halves of d for the scores (16-byte
//    loads of K rows), then D/2 dim pairs x (128 / (D/2)) key groups for
//    P V (coalesced bf16x2 loads of V rows).
//  * many small CTAs per SM keep many blocks in flight.
#include <cuda_bf16.h>

#include "seer_internal.h"
#include "seer_ptx.cuh"

namespace seer {

namespace {

constexpr int kDT = 128;             // threads per CTA
constexpr int kChunk = kDT;          // mask entries ranked per pass

__device__ __forceinline__ float exp2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int D>
__global__ void __launch_bounds__(kDT)
    decode_attn_kernel(const __nv_bfloat16 *__restrict__ q_tok, const __nv_bfloat16 *__restrict__ k,
                       const __nv_bfloat16 *__restrict__ v, const uint8_t *__restrict__ mask, int Hq, int Hkv, int L,
                       int nb, float scale_log2, int nsplit, float *__restrict__ part)
{
    constexpr int DH = D / 2;            // dims per thread in the score dot
    constexpr int NP = D / 2;            // dim pairs
    constexpr int KG = kDT / NP;         // key groups in P V (2 for d = 128, 4 for d = 64)
    constexpr int KPG = 64 / KG;         // keys per group
    __shared__ int s_list[kChunk];
    __shared__ int s_wsum[kDT / 32];
    __shared__ float s_red[kDT / 32];
    __shared__ float s_p[64];
    __shared__ float s_o[KG][D];
    const int split = blockIdx.x;
    const long long bh = blockIdx.y;
    const int b = (int)(bh / Hq), h = (int)(bh % Hq);
    const int kvh = h / (Hq / Hkv);
    const uint8_t *mrow = mask + bh * nb;
    const __nv_bfloat16 *kb = k + ((long long)b * Hkv + kvh) * L * D;
    const __nv_bfloat16 *vb = v + ((long long)b * Hkv + kvh) * L * D;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int kr = t >> 1, hf = t & 1;            // score role: key, half of d
    const int dp = t % NP, kg = t / NP;           // P V role: dim pair, key group

    float qv[DH];
    {
        const uint4 *qr = reinterpret_cast<const uint4 *>(q_tok + bh * D + hf * DH);
#pragma unroll
        for (int c = 0; c < DH / 8; ++c) {
            const uint4 u = qr[c];
            const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(p2[e]);
                qv[8 * c + 2 * e] = f.x;
                qv[8 * c + 2 * e + 1] = f.y;
            }
        }
    }
    float m = -INFINITY, l = 0.f, o0 = 0.f, o1 = 0.f;
    int rank_base = 0;
    for (int j0 = 0; j0 < nb; j0 += kChunk) {
        // Rank the active blocks of this chunk; keep those with rank = split (mod nsplit).
        const int j = j0 + t;
        const int a = (j < nb && mrow[j] != 0) ? 1 : 0;
        const unsigned bal = __ballot_sync(0xffffffffu, a);
        if (lane == 0)
            s_wsum[warp] = __popc(bal);
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kDT / 32; ++w) {
            before += w < warp ? s_wsum[w] : 0;
            total += s_wsum[w];
        }
        const int rank = rank_base + before + __popc(bal & ((1u << lane) - 1u));
        // this split's entries of the chunk, in rank order
        const int first = (rank_base % nsplit <= split) ? rank_base + (split - rank_base % nsplit)
                                                        : rank_base + nsplit - (rank_base % nsplit - split);
        if (a && (rank % nsplit) == split)
            s_list[(rank - first) / nsplit] = j;
        const int mine = (first < rank_base + total) ? (rank_base + total - 1 - first) / nsplit + 1 : 0;
        rank_base += total;
        __syncthreads();
        for (int e = 0; e < mine; ++e) {
            const int jb = s_list[e];
            // ---- scores of the block's 64 keys
            const int c = jb * 64 + kr;
            float s = 0.f;
            if (c < L) {
                const uint4 *kp = reinterpret_cast<const uint4 *>(kb + (long long)c * D + hf * DH);
#pragma unroll
                for (int cc = 0; cc < DH / 8; ++cc) {
                    const uint4 u = __ldg(kp + cc);
                    const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                    for (int ee = 0; ee < 4; ++ee) {
                        const float2 f = __bfloat1622float2(p2[ee]);
                        s = fmaf(qv[8 * cc + 2 * ee], f.x, fmaf(qv[8 * cc + 2 * ee + 1], f.y, s));
                    }
                }
            }
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s = (c < L) ? s * scale_log2 : -INFINITY;
            float wm = s;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1)
                wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, off));
            if (lane == 0)
                s_red[warp] = wm;
            __syncthreads();
            float bm = s_red[0];
#pragma unroll
            for (int w = 1; w < kDT / 32; ++w)
                bm = fmaxf(bm, s_red[w]);
            const float m_new = fmaxf(m, bm);        // finite: key 0 of every block exists
            const float alpha = exp2_approx(m - m_new);
            const float p = exp2_approx(s - m_new);
            if (hf == 0)
                s_p[kr] = p;
            __syncthreads();
            // ---- P V for this thread's dim pair over its key group
            float a0 = 0.f, a1 = 0.f, ls = 0.f;
#pragma unroll 4
            for (int q = 0; q < KPG; ++q) {
                const int key = kg * KPG + q;
                const int cc = jb * 64 + key;
                const float pk = s_p[key];
                ls += pk;
                if (cc < L) {
                    const float2 f = __bfloat1622float2(
                        *reinterpret_cast<const __nv_bfloat162 *>(vb + (long long)cc * D + 2 * dp));
                    a0 = fmaf(pk, f.x, a0);
                    a1 = fmaf(pk, f.y, a1);
                }
            }
            o0 = o0 * alpha + a0;
            o1 = o1 * alpha + a1;
            l = l * alpha + ls;                      // this key group's share of the row sum
            m = m_new;
            __syncthreads();                         // s_p / s_red are reused by the next block
        }
    }
    // Merge the key groups: o and l summed over groups (same m everywhere).
    s_o[kg][2 * dp] = o0;
    s_o[kg][2 * dp + 1] = o1;
    if (dp == 0)
        s_p[kg] = l;
    __syncthreads();
    float *out = part + (bh * nsplit + split) * (D + 2);
    for (int d = t; d < D; d += kDT) {
        float acc = 0.f;
#pragma unroll
        for (int g = 0; g < KG; ++g)
            acc += s_o[g][d];
        out[d] = acc;
    }
    if (t == 0) {
        float lt = 0.f;
#pragma unroll
        for (int g = 0; g < KG; ++g)
            lt += s_p[g];
        out[D] = m;
        out[D + 1] = lt;
    }
}


// ---------------------------------------------------------------------------
// GQA-group form (g = Hq/Hkv <= 8): one CTA per (kv head, split) serves all g
// query heads, so each K/V block crosses HBM -> SM once for the group.  The
// CTA walks the union of the heads' active blocks (a head that did not select
// a block gets p = 0 there and keeps its running max and sum: exact).  K and V
// blocks are staged in shared memory with cp.async, two blocks ahead.
constexpr int kGT = 256;             // threads
constexpr int kGMax = 8;             // heads per group served by this form

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int D>
__global__ void __launch_bounds__(kGT)
    decode_gqa_kernel(const __nv_bfloat16 *__restrict__ q_tok, const __nv_bfloat16 *__restrict__ k,
                      const __nv_bfloat16 *__restrict__ v, const uint8_t *__restrict__ mask, int Hq, int Hkv, int L,
                      int nb, float scale_log2, int nsplit, float *__restrict__ part)
{
    constexpr int RS = D + 8;                     // padded smem row (bf16): conflict-free 16-B reads
    constexpr int DQ = D / 4;                     // dims per thread in the score dot (4 dim quarters)
    constexpr int DPT = D / 32;                   // output dims per thread in P V
    extern __shared__ __align__(16) uint8_t gsm[];
    __nv_bfloat16 *sk = reinterpret_cast<__nv_bfloat16 *>(gsm);            // [2][64][RS]
    __nv_bfloat16 *sv = sk + 2 * 64 * RS;                                  // [2][64][RS]
    float *sq = reinterpret_cast<float *>(sv + 2 * 64 * RS);               // [kGMax][D]
    float *sred = sq + kGMax * D;                                          // [4][kGMax][64]
    float *sp = sred + 4 * kGMax * 64;                                     // [kGMax][64]
    float *salpha = sp + kGMax * 64;                                       // [kGMax]
    int *slist = reinterpret_cast<int *>(salpha + kGMax);                  // [kChunk] block | head bits << 16
    int *swsum = slist + kGT;                                              // [kGT / 32]
    const int split = blockIdx.x;
    const int bk = blockIdx.y;                                             // b * Hkv + kvh
    const int b = bk / Hkv, kvh = bk % Hkv;
    const int g = Hq / Hkv;
    const int h0 = kvh * g;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const __nv_bfloat16 *kb = k + (long long)bk * L * D;
    const __nv_bfloat16 *vb = v + (long long)bk * L * D;
    const uint8_t *mbase = mask + ((long long)b * Hq + h0) * nb;
    for (int e = t; e < g * D; e += kGT)
        sq[e] = __bfloat162float(q_tok[((long long)b * Hq + h0) * D + e]);

    // per-head online state: warp w < g owns head w's (m, l); every thread's
    // P V accumulators belong to head (t / 32)
    float m_h = -INFINITY, l_h = 0.f;
    float acc[DPT];
#pragma unroll
    for (int i = 0; i < DPT; ++i)
        acc[i] = 0.f;

    auto issue = [&](int stage, int jb) {
        // 64 rows of K and of V, D bf16 each: 64 * D / 8 16-byte pieces per tensor
        const uint32_t dk = smem_u32(sk + stage * 64 * RS), dv = smem_u32(sv + stage * 64 * RS);
        for (int e = t; e < 64 * D / 8; e += kGT) {
            const int r = e / (D / 8), c8 = e % (D / 8);
            const int row = jb * 64 + r;
            const bool ok = row < L;
            const long long off = (long long)(ok ? row : 0) * D + c8 * 8;
            cp_async16(dk + (uint32_t)(r * RS + c8 * 8) * 2, kb + off, ok ? 16 : 0);
            cp_async16(dv + (uint32_t)(r * RS + c8 * 8) * 2, vb + off, ok ? 16 : 0);
        }
    };

    int rank_base = 0;
    for (int j0 = 0; j0 < nb; j0 += kGT) {
        // union of the group's mask rows over this chunk, ranked; this split keeps rank = split (mod nsplit)
        const int j = j0 + t;
        int bitsj = 0;
        if (j < nb)
            for (int hh = 0; hh < g; ++hh)
                bitsj |= (mbase[(long long)hh * nb + j] != 0) << hh;
        const int a = bitsj != 0;
        const unsigned bal = __ballot_sync(0xffffffffu, a);
        if (lane == 0)
            swsum[warp] = __popc(bal);
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kGT / 32; ++w) {
            before += w < warp ? swsum[w] : 0;
            total += swsum[w];
        }
        const int rank = rank_base + before + __popc(bal & ((1u << lane) - 1u));
        const int r0 = rank_base % nsplit;
        const int first = rank_base + (split >= r0 ? split - r0 : nsplit - (r0 - split));
        if (a && (rank % nsplit) == split)
            slist[(rank - first) / nsplit] = j | (bitsj << 16);
        const int mine = (first < rank_base + total) ? (rank_base + total - 1 - first) / nsplit + 1 : 0;
        rank_base += total;
        __syncthreads();
        if (mine > 0)
            issue(0, slist[0] & 0xFFFF);
        cp_async_commit();
        if (mine > 1)
            issue(1, slist[1] & 0xFFFF);
        cp_async_commit();
        for (int e = 0; e < mine; ++e) {
            const int st = e & 1;
            const int jb = slist[e] & 0xFFFF;
            const int hbits = slist[e] >> 16;
            cp_async_wait<1>();                       // this block's group is complete
            __syncthreads();
            // ---- scores: thread = (key c, dim quarter dq), all g heads
            {
                const int c = t & 63, dq = t >> 6;
                const __nv_bfloat16 *kr = sk + (st * 64 + c) * RS + dq * DQ;
                float kf[DQ];
#pragma unroll
                for (int i = 0; i < DQ / 8; ++i) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(kr + 8 * i);
                    const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float2 f = __bfloat1622float2(p2[e2]);
                        kf[8 * i + 2 * e2] = f.x;
                        kf[8 * i + 2 * e2 + 1] = f.y;
                    }
                }
                for (int hh = 0; hh < g; ++hh) {
                    const float *qh = sq + hh * D + dq * DQ;
                    float s = 0.f;
#pragma unroll
                    for (int i = 0; i < DQ; ++i)
                        s = fmaf(qh[i], kf[i], s);
                    sred[(dq * kGMax + hh) * 64 + c] = s;
                }
            }
            __syncthreads();
            // ---- per-head online softmax: warp hh handles head hh
            if (warp < g) {
                const int hh = warp;
                const bool act = (hbits >> hh) & 1;
                float s0 = -INFINITY, s1 = -INFINITY;
                if (act) {
                    const int c0 = lane, c1 = lane + 32;
                    s0 = (sred[hh * 64 + c0] + sred[(kGMax + hh) * 64 + c0] + sred[(2 * kGMax + hh) * 64 + c0] +
                          sred[(3 * kGMax + hh) * 64 + c0]) * scale_log2;
                    s1 = (sred[hh * 64 + c1] + sred[(kGMax + hh) * 64 + c1] + sred[(2 * kGMax + hh) * 64 + c1] +
                          sred[(3 * kGMax + hh) * 64 + c1]) * scale_log2;
                    if (jb * 64 + c0 >= L)
                        s0 = -INFINITY;
                    if (jb * 64 + c1 >= L)
                        s1 = -INFINITY;
                }
                float bm = fmaxf(s0, s1);
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1)
                    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
                const float m_new = act ? fmaxf(m_h, bm) : m_h;
                const float alpha = act ? exp2_approx(m_h - m_new) : 1.0f;
                const float p0 = act ? exp2_approx(s0 - m_new) : 0.f;
                const float p1 = act ? exp2_approx(s1 - m_new) : 0.f;
                float ps = p0 + p1;
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1)
                    ps += __shfl_xor_sync(0xffffffffu, ps, off);
                sp[hh * 64 + lane] = p0;
                sp[hh * 64 + lane + 32] = p1;
                if (lane == 0)
                    salpha[hh] = alpha;
                l_h = l_h * alpha + ps;
                m_h = m_new;
            }
            __syncthreads();
            // ---- P V: warp hh accumulates head hh's output dims
            if (warp < g) {
                const int hh = warp;
                const float alpha = salpha[hh];
#pragma unroll
                for (int i = 0; i < DPT; ++i)
                    acc[i] *= alpha;
                const __nv_bfloat16 *vr = sv + st * 64 * RS + lane * DPT;
#pragma unroll 8
                for (int c = 0; c < 64; ++c) {
                    const float pc = sp[hh * 64 + c];
                    if (DPT == 4) {
                        const uint2 u = *reinterpret_cast<const uint2 *>(vr + c * RS);
                        const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
                        const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
                        acc[0] = fmaf(pc, f0.x, acc[0]);
                        acc[1] = fmaf(pc, f0.y, acc[1]);
                        acc[2 % DPT] = fmaf(pc, f1.x, acc[2 % DPT]);
                        acc[3 % DPT] = fmaf(pc, f1.y, acc[3 % DPT]);
                    } else {
                        const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(vr + c * RS));
                        acc[0] = fmaf(pc, f0.x, acc[0]);
                        acc[1 % DPT] = fmaf(pc, f0.y, acc[1 % DPT]);
                    }
                }
            }
            __syncthreads();                          // stage st is free again
            if (e + 2 < mine)
                issue(st, slist[e + 2] & 0xFFFF);
            cp_async_commit();
        }
        cp_async_wait<0>();
        __syncthreads();
    }
    // ---- partials of the g heads for this split
    if (warp < g) {
        const int hh = warp;
        float *out = part + (((long long)b * Hq + h0 + hh) * nsplit + split) * (D + 2);
#pragma unroll
        for (int i = 0; i < DPT; ++i)
            out[lane * DPT + i] = acc[i];
        if (lane == 0) {
            out[D] = m_h;
            out[D + 1] = l_h;
        }
    }
}

size_t gqa_smem_bytes(int D)
{
    return (size_t)2 * 2 * 64 * (D + 8) * 2 + sizeof(float) * ((size_t)kGMax * D + 4 * kGMax * 64 + kGMax * 64 +
                                                                  kGMax) +
           sizeof(int) * (kGT + kGT / 32);
}

// Merge the splits of one head: weights 2^(m_s - M), O = sum w o / sum w l.
template <int D>
__global__ void __launch_bounds__(D)
    decode_combine_kernel(const float *__restrict__ part, int nsplit, __nv_bfloat16 *__restrict__ o,
                          float *__restrict__ lse)
{
    // blockDim.x == D >= nsplit: thread s first reads split s's (m, l), the
    // block forms M and the weights, then thread c sums output dim c.
    __shared__ float sw[kMaxDecodeSplits];
    __shared__ float sred[2][D / 32];
    const long long bh = blockIdx.x;
    const float *pp = part + bh * nsplit * (D + 2);
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const float ms = t < nsplit ? pp[t * (D + 2) + D] : -INFINITY;
    const float ls = t < nsplit ? pp[t * (D + 2) + D + 1] : 0.f;
    float M = ms;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (lane == 0)
        sred[0][warp] = M;
    __syncthreads();
    M = sred[0][0];
#pragma unroll
    for (int w = 1; w < D / 32; ++w)
        M = fmaxf(M, sred[0][w]);
    const float w_s = (ms == -INFINITY || M == -INFINITY) ? 0.f : exp2_approx(ms - M);
    if (t < nsplit)
        sw[t] = w_s;
    float lt = w_s * ls;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        lt += __shfl_xor_sync(0xffffffffu, lt, off);
    if (lane == 0)
        sred[1][warp] = lt;
    __syncthreads();
    lt = 0.f;
#pragma unroll
    for (int w = 0; w < D / 32; ++w)
        lt += sred[1][w];
    // Every split's value of dim t first (all loads in flight together), then the
    // weighted sum in split order.
    float vals[kMaxDecodeSplits];
#pragma unroll
    for (int s2 = 0; s2 < kMaxDecodeSplits; ++s2)
        vals[s2] = s2 < nsplit ? pp[s2 * (D + 2) + t] : 0.f;
    float acc = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < kMaxDecodeSplits; ++s2)
        if (s2 < nsplit)
            acc = fmaf(sw[s2], vals[s2], acc);
    const bool has = lt > 0.f;
    o[bh * D + t] = __float2bfloat16(has ? acc / lt : 0.f);
    if (lse != nullptr && t == 0)
        lse[bh] = has ? (M + __log2f(lt)) * 0.69314718055994530942f : -INFINITY;
}

} // namespace

int decode_splits(int B, int Hq, int nb)
{
    return decode_splits_for(B, Hq, nb, 8);
}

// Splits so that about `per_sm` CTAs run per SM over `units` (heads, or KV
// heads for the group form); at most kMaxDecodeSplits and nb.
int decode_splits_for(int B, int units_per_b, int nb, int per_sm)
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
    const long long heads = (long long)B * units_per_b;
    long long s = ((long long)per_sm * sms + heads - 1) / heads;
    if (s > kMaxDecodeSplits)
        s = kMaxDecodeSplits;
    if (s > nb)
        s = nb;
    return (int)(s < 1 ? 1 : s);
}

// Splits of the group form: the smallest count whose grid fills at least 90 %
// of its last wave of resident CTAs (a grid of 1.08 waves ran 30 % slower than
// one of 0.97), else the best filling one; at most kMaxDecodeSplits and nb.
int gqa_splits(int units, int nb, int resident)
{
    const int cap = nb < kMaxDecodeSplits ? nb : kMaxDecodeSplits;
    int best = 1;
    double best_eff = -1.0;
    for (int ns = 1; ns <= cap; ++ns) {
        const long long ctas = (long long)units * ns;
        const long long waves = (ctas + resident - 1) / resident;
        const double eff = (double)ctas / (double)(waves * resident);
        if (eff >= 0.9)
            return ns;
        if (eff > best_eff) {
            best_eff = eff;
            best = ns;
        }
    }
    return best;
}

template <int D>
int gqa_resident_ctas(size_t smem)
{
    static int resident = 0;
    if (resident == 0) {
        int dev = 0, sms = 148, per_sm = 0;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_gqa_kernel<D>, kGT, smem) != cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
        resident = per_sm * sms;
    }
    return resident;
}

cudaError_t launch_decode(int B, int Hq, int Hkv, int L, int d, float scale_log2, const void *q_tok, const void *k,
                          const void *v, const uint8_t *mask, void *o, float *lse, float *part, cudaStream_t stream)
{
    const int nb = num_blocks(L);
    const int g = Hq / Hkv;
    const auto *qb = static_cast<const __nv_bfloat16 *>(q_tok);
    if (g <= kGMax && (d == 128 || d == 64)) {
        // group form: one CTA per (KV head, split)
        const size_t smem = gqa_smem_bytes(d);
        auto *ob = static_cast<__nv_bfloat16 *>(o);
        const auto *kb = static_cast<const __nv_bfloat16 *>(k);
        const auto *vb = static_cast<const __nv_bfloat16 *>(v);
        cudaError_t e = d == 128 ? cudaFuncSetAttribute(decode_gqa_kernel<128>,
                                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                                 : cudaFuncSetAttribute(decode_gqa_kernel<64>,
                                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        const int resident = d == 128 ? gqa_resident_ctas<128>(smem) : gqa_resident_ctas<64>(smem);
        const int ns = gqa_splits(B * Hkv, nb, resident);
        const dim3 grid(ns, B * Hkv);
        if (d == 128) {
            decode_gqa_kernel<128><<<grid, kGT, smem, stream>>>(qb, kb, vb, mask, Hq, Hkv, L, nb, scale_log2, ns, part);
            decode_combine_kernel<128><<<B * Hq, 128, 0, stream>>>(part, ns, ob, lse);
        } else {
            decode_gqa_kernel<64><<<grid, kGT, smem, stream>>>(qb, kb, vb, mask, Hq, Hkv, L, nb, scale_log2, ns, part);
            decode_combine_kernel<64><<<B * Hq, 64, 0, stream>>>(part, ns, ob, lse);
        }
        return cudaGetLastError();
    }
    const int ns = decode_splits(B, Hq, nb);
    const dim3 grid(ns, B * Hq);
    const auto *kb = static_cast<const __nv_bfloat16 *>(k);
    const auto *vb = static_cast<const __nv_bfloat16 *>(v);
    auto *ob = static_cast<__nv_bfloat16 *>(o);
    if (d == 128) {
        decode_attn_kernel<128><<<grid, kDT, 0, stream>>>(qb, kb, vb, mask, Hq, Hkv, L, nb, scale_log2, ns, part);
        decode_combine_kernel<128><<<B * Hq, 128, 0, stream>>>(part, ns, ob, lse);
    } else if (d == 64) {
        decode_attn_kernel<64><<<grid, kDT, 0, stream>>>(qb, kb, vb, mask, Hq, Hkv, L, nb, scale_log2, ns, part);
        decode_combine_kernel<64><<<B * Hq, 64, 0, stream>>>(part, ns, ob, lse);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

} // namespace seer
