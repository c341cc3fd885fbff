// seer_api.cu — the C ABI (include/seer.h): host-side argument checks,
// workspace sizing, tensor-map creation and kernel launches.  No device
// memory is ever allocated here; no host<->device copies are made except the
// status-word read in seer_check_status().
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/seer.h"
#include "seer_internal.h"
#include "seer_ptx.cuh"

namespace seer {

// Device status word: kernels record timeouts / failed checks here through a
// pointer (first error wins); seer_check_status() reads and clears it.
__device__ int g_status_word;

// Tile counters of the attention launches: a ring per device, one slot per
// launch, seeded on the launch stream.  256 launches can be in flight at once
// (on any number of streams) before a slot is reused; a kernel that finds its
// slot re-seeded by a later launch records kStatusRing (SEER_ERR_DEVICE).
constexpr int kTileCounterRing = 256;
__device__ unsigned long long g_tile_counters[kTileCounterRing];

namespace {

thread_local char g_err[512] = "";
unsigned long long g_timeout_ns = 2000000000ull;

seer_status fail(seer_status s, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return s;
}

seer_status ok()
{
    g_err[0] = '\0';
    return SEER_OK;
}

seer_status cuda_fail(cudaError_t e, const char *what)
{
    return fail(SEER_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

seer_status check_shape(const seer_shape *sh)
{
    if (sh == nullptr)
        return fail(SEER_ERR_INVALID_ARG, "shape is NULL");
    if (sh->B <= 0 || sh->Hq <= 0 || sh->Hkv <= 0 || sh->S <= 0 || sh->d <= 0)
        return fail(SEER_ERR_INVALID_ARG, "shape fields must be positive (B=%d Hq=%d Hkv=%d S=%d d=%d)", sh->B,
                    sh->Hq, sh->Hkv, sh->S, sh->d);
    if (sh->Hq % sh->Hkv != 0)
        return fail(SEER_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", sh->Hq, sh->Hkv);
    if (sh->d != 64 && sh->d != 128)
        return fail(SEER_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", sh->d);
    if (num_blocks(sh->S) > kMaxNb)
        return fail(SEER_ERR_UNSUPPORTED, "ceil(S/64) = %d exceeds %d", num_blocks(sh->S), kMaxNb);
    // B*Hq and B*Hkv index a grid dimension of at most 65535 in the decode and
    // gate kernels (and B*Hq*nb stays below 2^30).
    if ((long long)sh->B * sh->Hq > 65535)
        return fail(SEER_ERR_UNSUPPORTED, "B*Hq = %lld exceeds 65535", (long long)sh->B * sh->Hq);
    return SEER_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int *status_ptr()
{
    // One address per device (the symbol lives in each device's copy of the module).
    static std::mutex mu;
    static int *cache[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess)
            return nullptr;
        cache[dev] = static_cast<int *>(p);
    }
    return cache[dev];
}

// A tile counter for one attention launch: the next slot of this device's
// ring, seeded on `stream` before the launch with a byte pattern (*base) that
// changes every time the slot comes round again.  Null on a CUDA error (in *err).
unsigned long long *tile_counter(cudaStream_t stream, cudaError_t *err, unsigned long long *base)
{
    static std::mutex mu;
    static unsigned long long *cache[64] = {nullptr};
    static unsigned next[64] = {0};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess)
        return nullptr;
    if (dev < 0 || dev >= 64) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    unsigned long long *c = nullptr;
    int tag = 1;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (cache[dev] == nullptr) {
            void *ptr = nullptr;
            *err = cudaGetSymbolAddress(&ptr, g_tile_counters);
            if (*err != cudaSuccess)
                return nullptr;
            cache[dev] = static_cast<unsigned long long *>(ptr);
        }
        const unsigned seq = next[dev]++;
        c = cache[dev] + (seq % kTileCounterRing);
        tag = (int)((seq / kTileCounterRing) % 255u) + 1;
    }
    *base = 0x0101010101010101ull * (unsigned long long)tag;
    *err = cudaMemsetAsync(c, tag, sizeof(unsigned long long), stream);
    return *err == cudaSuccess ? c : nullptr;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

} // namespace

seer_status set_last_error(seer_status s, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return s;
}

// [B*H, S, d] bf16 viewed as a 3D tensor (d innermost); 64 x 64 boxes with
// the 128-byte swizzle the MMA descriptors expect.
bool make_tmap_bhsd(CUtensorMap *map, const void *base, int BH, int S, int d)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr)
        return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)S, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)S * d * 2};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// [B*H, S, d] bf16 viewed as 4-D (64 columns, S rows, d/64 panels, B*H) so
// that one 64-row box brings every 64-column panel of a block at once,
// panel-major, each panel in the 128-byte swizzle layout.
bool make_tmap_bhsd_panels(CUtensorMap *map, const void *base, int BH, int S, int d)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr)
        return false;
    const cuuint64_t dims[4] = {64, (cuuint64_t)S, (cuuint64_t)(d / 64), (cuuint64_t)BH};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, 128, (cuuint64_t)S * d * 2};
    const cuuint32_t box[4] = {64, 64, (cuuint32_t)(d / 64), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

} // namespace seer

using namespace seer;

extern "C" {

const char *seer_version(void) { return "seer-b200 0.1.0 (sm_100a)"; }

const char *seer_last_error(void) { return g_err; }

void seer_set_wait_timeout_ns(unsigned long long ns) { g_timeout_ns = ns; }

size_t seer_workspace_bytes(int which_call, const seer_shape *shape)
{
    if (check_shape(shape) != SEER_OK)
        return 0;
    const int nb = num_blocks(shape->S);
    switch (which_call) {
    case SEER_CALL_GATE_SCORES:
        return gate_workspace_bytes(shape->B, shape->Hq, shape->Hkv, shape->S, shape->d, 256, true);
    case SEER_CALL_BLOCK_SPARSE_PREFILL:
        return 0;
    case SEER_CALL_ATTN_POOLED_MAP:
        return sizeof(float) * (size_t)kMaxAttnCtas * nb * 128;
    case SEER_CALL_DECODE_GATE_SCORES:
        return decode_gate_ws_bytes(shape->B, shape->Hq, shape->Hkv, shape->S, shape->d, 256, true);
    case SEER_CALL_GATE_KEY_CACHE:
        return gate_key_ws_bytes(shape->B, shape->Hkv, shape->S, shape->d, true);
    case SEER_CALL_DECODE_GATE_CACHED:
        return ((sizeof(float) * (size_t)shape->B * shape->Hq * shape->d + 255) & ~size_t(255)) +
               ((sizeof(float) * (size_t)shape->B * shape->Hq * 256 + 255) & ~size_t(255));
    case SEER_CALL_BLOCK_SPARSE_DECODE:
        return sizeof(float) * (size_t)shape->B * shape->Hq * kMaxDecodeSplits * (shape->d + 2);
    default:
        fail(SEER_ERR_INVALID_ARG, "unknown call id %d", which_call);
        return 0;
    }
}

// Argument checks shared by the prefill and decode gates.
// need_kind: 0 = the prefill gate's workspace, 1 = the decode gate's, 2 = the
// key-cache call's, 3 = the cached decode row's.
static seer_status check_gate_args(const char *name, const seer_shape *shape, const void *q, const void *k,
                                   const void *wq, const void *wk, const seer_gate_params *gp, const float *scores,
                                   void *workspace, size_t ws_bytes, int need_kind = 0)
{
    seer_status st = check_shape(shape);
    if (st != SEER_OK)
        return st;
    if (gp == nullptr || q == nullptr || k == nullptr || wq == nullptr || wk == nullptr || scores == nullptr)
        return fail(SEER_ERR_INVALID_ARG, "%s: NULL argument", name);
    if (gp->d_gate < 2 || gp->d_gate > 256 || (gp->d_gate & 1))
        return fail(SEER_ERR_UNSUPPORTED, "d_gate %d must be even and in [2, 256]", gp->d_gate);
    if (!(gp->rope_theta > 0.f) || !std::isfinite(gp->rope_theta))
        return fail(SEER_ERR_INVALID_ARG, "rope_theta must be positive and finite");
    if (gp->wq_head_stride < 0 || gp->wk_head_stride < 0)
        return fail(SEER_ERR_INVALID_ARG, "weight head strides must be >= 0");
    if (!aligned16(q) || !aligned16(k))
        return fail(SEER_ERR_INVALID_ARG, "q and k must be 16-byte aligned");
    if ((gp->d_gate % 4) != 0)
        return fail(SEER_ERR_UNSUPPORTED, "d_gate %d must be a multiple of 4", gp->d_gate);
    if (gp->k_pooling != SEER_KPOOL_AVG && gp->k_pooling != SEER_KPOOL_MAXMIN)
        return fail(SEER_ERR_INVALID_ARG, "unknown k_pooling %d", gp->k_pooling);
    const bool maxmin = gp->k_pooling == SEER_KPOOL_MAXMIN;
    if (gate_projection_smem(maxmin ? 2 * shape->d : shape->d, gp->d_gate) > 227 * 1024)
        return fail(SEER_ERR_UNSUPPORTED, "d_gate %d too large for %s K pooling at d = %d", gp->d_gate,
                    maxmin ? "max+min" : "average", shape->d);
    size_t need = gate_workspace_bytes(shape->B, shape->Hq, shape->Hkv, shape->S, shape->d, gp->d_gate, maxmin);
    if (need_kind == 1)
        need = decode_gate_ws_bytes(shape->B, shape->Hq, shape->Hkv, shape->S, shape->d, gp->d_gate, maxmin);
    else if (need_kind == 2)
        need = gate_key_ws_bytes(shape->B, shape->Hkv, shape->S, shape->d, maxmin);
    else if (need_kind == 3)   // the token's q rows, fp32, before and after the projection
        need = ((sizeof(float) * (size_t)shape->B * shape->Hq * shape->d + 255) & ~size_t(255)) +
               ((sizeof(float) * (size_t)shape->B * shape->Hq * gp->d_gate + 255) & ~size_t(255));
    if (workspace == nullptr || ws_bytes < need)
        return fail(SEER_ERR_WORKSPACE, "%s needs %zu workspace bytes, got %zu", name, need, ws_bytes);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(SEER_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    return SEER_OK;
}

seer_status seer_gate_scores(const seer_shape *shape, const void *q, const void *k, const void *wq, const void *wk,
                             const seer_gate_params *gp, float *scores, void *workspace, size_t ws_bytes,
                             void *stream)
{
    const seer_status st = check_gate_args("seer_gate_scores", shape, q, k, wq, wk, gp, scores, workspace, ws_bytes);
    if (st != SEER_OK)
        return st;
    const bool maxmin = gp->k_pooling == SEER_KPOOL_MAXMIN;
    const cudaError_t e = launch_gate(shape->B, shape->Hq, shape->Hkv, shape->S, shape->d, gp->d_gate,
                                      gp->rope_theta, maxmin, q, k, wq, gp->wq_head_stride, wk, gp->wk_head_stride,
                                      scores, workspace, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_gate_scores launch");
    return ok();
}

seer_status seer_block_mask(const seer_shape *shape, const float *scores, const seer_mask_params *mp, uint8_t *mask,
                            void *stream)
{
    seer_status st = check_shape(shape);
    if (st != SEER_OK)
        return st;
    if (mp == nullptr || scores == nullptr || mask == nullptr)
        return fail(SEER_ERR_INVALID_ARG, "seer_block_mask: NULL argument");
    if (mp->mode != SEER_MASK_THRESHOLD && mp->mode != SEER_MASK_TOPK)
        return fail(SEER_ERR_INVALID_ARG, "unknown mask mode %d", mp->mode);
    if (mp->mode == SEER_MASK_TOPK && mp->k_per_row == nullptr && mp->k_fixed <= 0 &&
        !(std::isfinite(mp->density) && mp->density >= 0.0))
        return fail(SEER_ERR_INVALID_ARG, "TopK density must be finite and >= 0");
    if (mp->mode == SEER_MASK_THRESHOLD && std::isnan(mp->threshold))
        return fail(SEER_ERR_INVALID_ARG, "threshold is NaN");
    const cudaError_t e = launch_mask(shape->B, shape->Hq, num_blocks(shape->S), scores, mp->mode, mp->threshold,
                                      mp->density, mp->k_fixed, mp->k_per_row, mp->force_first ? 1 : 0,
                                      mp->force_diag ? 1 : 0, mask, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_block_mask launch");
    return ok();
}

seer_status seer_compact_mask(const seer_shape *shape, const uint8_t *mask, int32_t *lists, int32_t *counts,
                              void *stream)
{
    seer_status st = check_shape(shape);
    if (st != SEER_OK)
        return st;
    if (mask == nullptr || lists == nullptr || counts == nullptr)
        return fail(SEER_ERR_INVALID_ARG, "seer_compact_mask: NULL argument");
    const cudaError_t e =
        launch_compact(shape->B, shape->Hq, num_blocks(shape->S), mask, lists, counts, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_compact_mask launch");
    return ok();
}

static seer_status attention_common(const char *name, const seer_shape *shape, const void *q, const void *k,
                                    const void *v, void *o)
{
    seer_status st = check_shape(shape);
    if (st != SEER_OK)
        return st;
    if (q == nullptr || k == nullptr || v == nullptr || o == nullptr)
        return fail(SEER_ERR_INVALID_ARG, "%s: NULL q/k/v/o", name);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(SEER_ERR_INVALID_ARG, "%s: q, k, v, o must be 16-byte aligned", name);
    return SEER_OK;
}

seer_status seer_block_sparse_prefill(const seer_shape *shape, const void *q, const void *k, const void *v,
                                      const uint8_t *mask, float softmax_scale, void *o, float *lse, void *workspace,
                                      size_t ws_bytes, void *stream)
{
    (void)workspace;
    (void)ws_bytes;
    seer_status st = attention_common("seer_block_sparse_prefill", shape, q, k, v, o);
    if (st != SEER_OK)
        return st;
    if (mask == nullptr)
        return fail(SEER_ERR_INVALID_ARG, "seer_block_sparse_prefill: NULL mask");
    if (std::isnan(softmax_scale) || std::isinf(softmax_scale))
        return fail(SEER_ERR_INVALID_ARG, "softmax_scale must be finite");
    int *status = status_ptr();
    if (status == nullptr)
        return fail(SEER_ERR_CUDA, "cannot resolve the device status word");
    AttnLaunch a{};
    a.B = shape->B;
    a.Hq = shape->Hq;
    a.Hkv = shape->Hkv;
    a.S = shape->S;
    a.d = shape->d;
    a.nb = num_blocks(shape->S);
    const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)shape->d);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.mask = mask;
    a.o = o;
    a.lse = lse;
    a.q = q;
    a.k = k;
    a.v = v;
    a.map_mode = false;
    a.timeout_ns = g_timeout_ns;
    a.status = status;
    cudaError_t e = cudaSuccess;
    a.tile_ctr = tile_counter(static_cast<cudaStream_t>(stream), &e, &a.tile_base);
    if (a.tile_ctr == nullptr)
        return cuda_fail(e, "seer_block_sparse_prefill tile counter");
    e = launch_attention(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_block_sparse_prefill launch");
    return ok();
}

seer_status seer_attn_pooled_map(const seer_shape *shape, const void *q, const void *k, const void *v,
                                 float softmax_scale, void *o, float *A, void *workspace, size_t ws_bytes,
                                 void *stream)
{
    seer_status st = attention_common("seer_attn_pooled_map", shape, q, k, v, o);
    if (st != SEER_OK)
        return st;
    if (A == nullptr)
        return fail(SEER_ERR_INVALID_ARG, "seer_attn_pooled_map: NULL A");
    if (std::isnan(softmax_scale) || std::isinf(softmax_scale))
        return fail(SEER_ERR_INVALID_ARG, "softmax_scale must be finite");
    const int nb = num_blocks(shape->S);
    const int grid = attn_grid_size(shape->B, shape->Hq, shape->Hkv, nb);
    const size_t need = sizeof(float) * (size_t)grid * nb * 128;
    if (workspace == nullptr || ws_bytes < need)
        return fail(SEER_ERR_WORKSPACE, "seer_attn_pooled_map needs %zu workspace bytes, got %zu", need, ws_bytes);
    int *status = status_ptr();
    if (status == nullptr)
        return fail(SEER_ERR_CUDA, "cannot resolve the device status word");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(A, 0, sizeof(float) * (size_t)shape->B * shape->Hq * nb * nb, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_attn_pooled_map memset");
    AttnLaunch a{};
    a.B = shape->B;
    a.Hq = shape->Hq;
    a.Hkv = shape->Hkv;
    a.S = shape->S;
    a.d = shape->d;
    a.nb = nb;
    const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)shape->d);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.o = o;
    a.A = A;
    a.rscratch = static_cast<float *>(workspace);
    a.q = q;
    a.k = k;
    a.v = v;
    a.map_mode = true;
    a.timeout_ns = g_timeout_ns;
    a.status = status;
    a.tile_ctr = tile_counter(s, &e, &a.tile_base);
    if (a.tile_ctr == nullptr)
        return cuda_fail(e, "seer_attn_pooled_map tile counter");
    e = launch_attention(a, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_attn_pooled_map launch");
    return ok();
}

seer_status seer_distill_loss(const seer_shape *shape, const float *scores, const float *A, float *A_norm,
                              float *loss_rows, float *loss, void *stream)
{
    seer_status st = check_shape(shape);
    if (st != SEER_OK)
        return st;
    if (scores == nullptr || A == nullptr || loss_rows == nullptr || loss == nullptr)
        return fail(SEER_ERR_INVALID_ARG, "seer_distill_loss: NULL scores, A, loss_rows or loss");
    const cudaError_t e = launch_distill(shape->B, shape->Hq, num_blocks(shape->S), scores, A, A_norm, loss_rows, loss,
                                         static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_distill_loss launch");
    return ok();
}

seer_status seer_check_status(void *stream)
{
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_check_status sync");
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_status_word, sizeof(int));
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_check_status read");
    if (v != 0) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int));
        if (v == kStatusTimeout)
            return fail(SEER_ERR_TIMEOUT, "a device-side wait ran out");
        if (v == kStatusRing)
            return fail(SEER_ERR_DEVICE, "more than 256 attention launches were in flight at once: a tile-counter "
                                         "slot was reused by a later launch (outputs of the earlier one are incomplete)");
        if (v == kStatusSmem)
            return fail(SEER_ERR_DEVICE, "the attention kernel's shared-memory layout did not fit its window once "
                                         "aligned (no output was written)");
        return fail(SEER_ERR_DEVICE, "device-side check failed (code %d)", v);
    }
    return ok();
}

// ---------------------------------------------------------------- decode step
seer_status seer_decode_gate_scores(const seer_shape *shape, const void *q_tok, const void *k, const void *wq,
                                    const void *wk, const seer_gate_params *gp, float *scores, void *workspace,
                                    size_t ws_bytes, void *stream)
{
    const seer_status st =
        check_gate_args("seer_decode_gate_scores", shape, q_tok, k, wq, wk, gp, scores, workspace, ws_bytes, 1);
    if (st != SEER_OK)
        return st;
    if (num_blocks(shape->S) * sizeof(float) + 1024 > 227 * 1024)
        return fail(SEER_ERR_UNSUPPORTED, "seer_decode_gate_scores: nb = %d too large", num_blocks(shape->S));
    const cudaError_t e = launch_decode_gate(shape->B, shape->Hq, shape->Hkv, shape->S, shape->d, gp->d_gate,
                                             gp->rope_theta, gp->k_pooling == SEER_KPOOL_MAXMIN, q_tok, k, wq,
                                             gp->wq_head_stride, wk, gp->wk_head_stride, scores, workspace,
                                             static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_decode_gate_scores launch");
    return ok();
}

seer_status seer_gate_key_cache(const seer_shape *shape, const void *k, const void *wk, const seer_gate_params *gp,
                                int first_block, float *kt, void *workspace, size_t ws_bytes, void *stream)
{
    // the q and wq checks of the shared helper are satisfied with k and wk
    const seer_status st =
        check_gate_args("seer_gate_key_cache", shape, k, k, wk, wk, gp, kt, workspace, ws_bytes, 2);
    if (st != SEER_OK)
        return st;
    if (first_block < 0 || first_block > num_blocks(shape->S))
        return fail(SEER_ERR_INVALID_ARG, "first_block %d outside [0, %d]", first_block, num_blocks(shape->S));
    const cudaError_t e = launch_gate_keys(shape->B, shape->Hkv, shape->S, shape->d, gp->d_gate, gp->rope_theta,
                                           gp->k_pooling == SEER_KPOOL_MAXMIN, k, wk, gp->wk_head_stride, first_block,
                                           kt, workspace, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_gate_key_cache launch");
    return ok();
}

seer_status seer_decode_gate_scores_cached(const seer_shape *shape, const void *q_tok, const float *kt,
                                           const void *wq, const seer_gate_params *gp, float *scores, void *workspace,
                                           size_t ws_bytes, void *stream)
{
    const seer_status st = check_gate_args("seer_decode_gate_scores_cached", shape, q_tok, kt, wq, wq, gp, scores,
                                           workspace, ws_bytes, 3);
    if (st != SEER_OK)
        return st;
    if ((reinterpret_cast<uintptr_t>(kt) & 15u) != 0)
        return fail(SEER_ERR_INVALID_ARG, "kt must be 16-byte aligned");
    const cudaError_t e = launch_decode_gate_cached(shape->B, shape->Hq, shape->Hkv, shape->S, shape->d, gp->d_gate,
                                                    gp->rope_theta, q_tok, wq, gp->wq_head_stride, kt, scores,
                                                    workspace, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_decode_gate_scores_cached launch");
    return ok();
}

seer_status seer_topk_from_density(double density, int nb, int force_first, int force_diag, int32_t *k_out)
{
    if (k_out == nullptr)
        return fail(SEER_ERR_INVALID_ARG, "seer_topk_from_density: NULL k_out");
    if (nb < 1 || nb > kMaxNb)
        return fail(SEER_ERR_INVALID_ARG, "seer_topk_from_density: nb = %d outside [1, %d]", nb, kMaxNb);
    if (!(std::isfinite(density) && density >= 0.0))
        return fail(SEER_ERR_INVALID_ARG, "seer_topk_from_density: density must be finite and >= 0");
    for (int i = 0; i < nb; ++i) {
        // The rule of the TopK mask kernels: ceil(density * (i + 1)) in double,
        // clamped to [#forced, i + 1] (block 0 and the diagonal coincide in row 0).
        const int n_forced = (force_first ? 1 : 0) + ((force_diag && !(force_first && i == 0)) ? 1 : 0);
        const double want = std::ceil(density * (double)(i + 1));
        int k = want > (double)(i + 1) ? i + 1 : (int)want;
        if (k < n_forced)
            k = n_forced;
        if (k > i + 1)
            k = i + 1;
        k_out[i] = k;
    }
    return ok();
}

seer_status seer_decode_block_mask(const seer_shape *shape, const float *scores, const seer_mask_params *mp,
                                   uint8_t *mask, void *stream)
{
    seer_status st = check_shape(shape);
    if (st != SEER_OK)
        return st;
    if (mp == nullptr || scores == nullptr || mask == nullptr)
        return fail(SEER_ERR_INVALID_ARG, "seer_decode_block_mask: NULL argument");
    if (mp->mode != SEER_MASK_THRESHOLD && mp->mode != SEER_MASK_TOPK)
        return fail(SEER_ERR_INVALID_ARG, "unknown mask mode %d", mp->mode);
    if (mp->mode == SEER_MASK_TOPK && mp->k_per_row == nullptr && mp->k_fixed <= 0 &&
        !(std::isfinite(mp->density) && mp->density >= 0.0))
        return fail(SEER_ERR_INVALID_ARG, "TopK density must be finite and >= 0");
    if (mp->mode == SEER_MASK_THRESHOLD && std::isnan(mp->threshold))
        return fail(SEER_ERR_INVALID_ARG, "threshold is NaN");
    const int nb = num_blocks(shape->S);
    const cudaError_t e = launch_mask_rows(shape->B, shape->Hq, nb, 1, nb - 1, scores, mp->mode, mp->threshold,
                                           mp->density, mp->k_fixed, mp->k_per_row, mp->force_first ? 1 : 0,
                                           mp->force_diag ? 1 : 0, mask, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_decode_block_mask launch");
    return ok();
}

seer_status seer_block_sparse_decode(const seer_shape *shape, const void *q_tok, const void *k, const void *v,
                                     const uint8_t *mask, float softmax_scale, void *o, float *lse, void *workspace,
                                     size_t ws_bytes, void *stream)
{
    seer_status st = attention_common("seer_block_sparse_decode", shape, q_tok, k, v, o);
    if (st != SEER_OK)
        return st;
    if (mask == nullptr)
        return fail(SEER_ERR_INVALID_ARG, "seer_block_sparse_decode: NULL mask");
    if (std::isnan(softmax_scale) || std::isinf(softmax_scale))
        return fail(SEER_ERR_INVALID_ARG, "softmax_scale must be finite");
    const size_t need = seer_workspace_bytes(SEER_CALL_BLOCK_SPARSE_DECODE, shape);
    if (workspace == nullptr || ws_bytes < need)
        return fail(SEER_ERR_WORKSPACE, "seer_block_sparse_decode needs %zu workspace bytes, got %zu", need,
                    ws_bytes);
    if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
        return fail(SEER_ERR_WORKSPACE, "workspace must be 16-byte aligned");
    const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)shape->d);
    const cudaError_t e =
        launch_decode(shape->B, shape->Hq, shape->Hkv, shape->S, shape->d, scale * 1.4426950408889634f, q_tok, k, v,
                      mask, o, lse, static_cast<float *>(workspace), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "seer_block_sparse_decode launch");
    return ok();
}

} // extern "C"
