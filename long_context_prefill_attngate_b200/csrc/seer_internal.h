// seer_internal.h — declarations shared by the library's .cu files (host side).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/seer.h"

namespace seer {

constexpr int kBlock = 64;            // block size of gate, mask and kernels

// Blocks of a sequence of S tokens; the last one holds S - 64 (nb - 1) tokens
// when S is not a multiple of 64.
inline int num_blocks(int S) { return (S + kBlock - 1) / kBlock; }
constexpr int kMaxNb = 16384;         // S <= 1M tokens
constexpr int kMaxAttnCtas = 296;     // tile pipelines in flight: 2 slots x 148 SMs
constexpr int kAttnThreads = 512;     // 2 slots x (4 softmax + Q/K producer + MMA + list builder + V producer) warps

struct AttnLaunch {
    int B, Hq, Hkv, S, d, nb;
    float scale_log2;             // softmax scale * log2(e)
    const uint8_t *mask;          // sparse mode: [B,Hq,nb,nb]
    void *o;                      // bf16 [B,Hq,S,d]
    float *lse;                   // fp32 [B,Hq,S] or null
    float *A;                     // map mode: fp32 [B,Hq,nb,nb]
    float *rscratch;              // map mode: [grid][nb][128]
    const void *q, *k, *v;
    bool map_mode;
    uint64_t timeout_ns;
    int *status;                  // device status word
    unsigned long long *tile_ctr; // tile counter of this launch, seeded with tile_base on the launch stream
    unsigned long long tile_base;
};

// Attention kernels (seer_attn.cu).  Returns a cudaError_t.
cudaError_t launch_attention(const AttnLaunch &p, cudaStream_t stream);
// Block-sparse prefill with one head's query block per tile (seer_sparse.cu).
cudaError_t launch_sparse_attention(const AttnLaunch &p, cudaStream_t stream);
int attn_grid_size(int B, int Hq, int Hkv, int nb);

// Gate kernels (seer_gate.cu).
cudaError_t launch_gate(int B, int Hq, int Hkv, int S, int d, int dg, float theta, bool k_maxmin, const void *q,
                        const void *k, const void *wq, long long wq_stride, const void *wk, long long wk_stride,
                        float *scores, void *ws, cudaStream_t stream);
size_t gate_workspace_bytes(int B, int Hq, int Hkv, int S, int d, int dg, bool k_maxmin);
size_t gate_projection_smem(int d_in, int dg);
cudaError_t launch_decode_gate(int B, int Hq, int Hkv, int L, int d, int dg, float theta, bool k_maxmin,
                               const void *q_tok, const void *k, const void *wq, long long wq_stride, const void *wk,
                               long long wk_stride, float *scores, void *ws, cudaStream_t stream);
cudaError_t launch_gate_keys(int B, int Hkv, int L, int d, int dg, float theta, bool k_maxmin, const void *k,
                             const void *wk, long long wk_stride, int first_block, float *kt, void *ws,
                             cudaStream_t stream);
cudaError_t launch_decode_gate_cached(int B, int Hq, int Hkv, int L, int d, int dg, float theta, const void *q_tok,
                                      const void *wq, long long wq_stride, const float *kt, float *scores, void *ws,
                                      cudaStream_t stream);
size_t gate_key_ws_bytes(int B, int Hkv, int L, int d, bool k_maxmin);
size_t decode_gate_ws_bytes(int B, int Hq, int Hkv, int L, int d, int dg, bool k_maxmin);

// Block-sparse decode attention (seer_decode.cu).
constexpr int kMaxDecodeSplits = 64;
int decode_splits(int B, int Hq, int nb);
int decode_splits_for(int B, int units_per_b, int nb, int per_sm);
cudaError_t launch_decode(int B, int Hq, int Hkv, int L, int d, float scale_log2, const void *q_tok, const void *k,
                          const void *v, const uint8_t *mask, void *o, float *lse, float *part, cudaStream_t stream);

// Mask / compaction kernels (seer_mask.cu).
cudaError_t launch_mask(int B, int Hq, int nb, const float *scores, int mode, float threshold,
                        double density, int k_fixed, const int32_t *k_per_row, int force_first,
                        int force_diag, uint8_t *mask, cudaStream_t stream);
cudaError_t launch_mask_rows(int B, int Hq, int nb, int R, int i0, const float *scores, int mode, float threshold,
                             double density, int k_fixed, const int32_t *k_per_row, int ff, int fd, uint8_t *mask,
                             cudaStream_t stream);
cudaError_t launch_compact(int B, int Hq, int nb, const uint8_t *mask, int32_t *lists, int32_t *counts,
                           cudaStream_t stream);

// Distillation target and loss (seer_distill.cu).
cudaError_t launch_distill(int B, int Hq, int nb, const float *G, const float *A, float *ahat, float *loss_rows,
                           float *loss, cudaStream_t stream);

// Record the thread-local error text returned by seer_last_error() (seer_api.cu).
seer_status set_last_error(seer_status s, const char *fmt, ...);

// Tensor-map creation through the driver entry point (seer_api.cu).
bool make_tmap_bhsd(CUtensorMap *map, const void *base, int BH, int S, int d);
bool make_tmap_bhsd_panels(CUtensorMap *map, const void *base, int BH, int S, int d);

} // namespace seer
