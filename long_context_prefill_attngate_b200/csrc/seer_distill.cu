// seer_distill.cu — the AttnGate distillation target and loss.
//
// "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs", rebuttal
// Question 2: the max-pooled attention map is row-normalised so it matches the
// gate's softmax output (rows sum to 1); Q2 on the loss: the gate is trained
// with an MSE loss against that target.  For soft scores G and map A
// (fp32 [B, Hq, nb, nb]):
//   Ahat[i, j]      = A[i, j] / sum_{j' <= i} A[i, j']   (0 for j > i; a zero row stays 0)
//   loss_rows[b,h,i] = sum_{j <= i} (G[i, j] - Ahat[i, j])^2
//   loss[b, h]      = sum_i loss_rows[b, h, i] / (nb (nb + 1) / 2)
// Both reductions run in a fixed order, so results are bit-reproducible.
// HBM bound: G and A read once, Ahat (optional) written once.
#include "seer_internal.h"

namespace seer {

namespace {

constexpr int kRowWarps = 8;

__global__ void __launch_bounds__(kRowWarps * 32)
    distill_rows_kernel(const float *__restrict__ G, const float *__restrict__ A, long long rows, int nb,
                        float *__restrict__ ahat, float *__restrict__ loss_rows)
{
    const long long row = (long long)blockIdx.x * kRowWarps + (threadIdx.x >> 5);
    if (row >= rows)
        return;
    const int lane = threadIdx.x & 31;
    const int i = (int)(row % nb);
    const float *a = A + row * nb;
    const float *g = G + row * nb;
    float s = 0.f;
    for (int j = lane; j <= i; j += 32)
        s += a[j];
#pragma unroll
    for (int off = 16; off; off >>= 1)
        s += __shfl_xor_sync(0xffffffffu, s, off);
    const float inv = s > 0.f ? 1.0f / s : 0.f;
    float l = 0.f;
    for (int j = lane; j < nb; j += 32) {
        const float t = j <= i ? a[j] * inv : 0.f;
        if (ahat != nullptr)
            ahat[row * nb + j] = t;
        if (j <= i) {
            const float dlt = g[j] - t;
            l = fmaf(dlt, dlt, l);
        }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1)
        l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0)
        loss_rows[row] = l;
}

constexpr int kHeadThreads = 256;

__global__ void __launch_bounds__(kHeadThreads)
    distill_heads_kernel(const float *__restrict__ loss_rows, int nb, float *__restrict__ loss)
{
    __shared__ float part[kHeadThreads];
    const long long bh = blockIdx.x;
    float s = 0.f;
    for (int i = threadIdx.x; i < nb; i += kHeadThreads)
        s += loss_rows[bh * nb + i];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = kHeadThreads / 2; w > 0; w >>= 1) {
        if (threadIdx.x < w)
            part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0)
        loss[bh] = part[0] / (0.5f * (float)nb * (float)(nb + 1));
}

} // namespace

cudaError_t launch_distill(int B, int Hq, int nb, const float *G, const float *A, float *ahat, float *loss_rows,
                           float *loss, cudaStream_t stream)
{
    const long long rows = (long long)B * Hq * nb;
    distill_rows_kernel<<<(unsigned)((rows + kRowWarps - 1) / kRowWarps), kRowWarps * 32, 0, stream>>>(
        G, A, rows, nb, ahat, loss_rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    distill_heads_kernel<<<(unsigned)((long long)B * Hq), kHeadThreads, 0, stream>>>(loss_rows, nb, loss);
    return cudaGetLastError();
}

} // namespace seer
