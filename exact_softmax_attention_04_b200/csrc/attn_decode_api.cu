// attn_decode_api.cu - host side of the decode step against rolling caches:
// argument checks, split choice, workspace layout, TMA descriptors, the two
// launches. Contracts in include/attn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>

#include "attn.h"
#include "attn_decode_kernel.cuh"
#include "attn_host.h"

namespace {

using namespace attn_host;

bool g_dec_set[kMaxDevices][2][5] = {};  // [device][d==128][log2 NC]

// Splits of the W slots per (batch, kv head): whole 128-slot tiles, two
// resident CTAs per SM of a 148-SM B200. Minimises waves x (tiles per split
// + 1), the +1 standing for a CTA's pipeline fill and drain.
void choose_splits(int64_t bkv, int W, int *nsplit, int *chunk)
{
    const int tiles = (W + attn_sm100::DEC_TK - 1) / attn_sm100::DEC_TK;
    const int64_t resident = 2 * 148;
    int best_per = tiles;
    double best_cost = -1.0;
    for (int ns = 1; ns <= tiles && ns <= 64; ++ns) {
        const int per = (tiles + ns - 1) / ns;
        const int64_t ctas = bkv * ((tiles + per - 1) / per);
        const double cost = static_cast<double>((ctas + resident - 1) / resident) * (per + 1.0);
        if (best_cost < 0.0 || cost < best_cost) {
            best_cost = cost;
            best_per = per;
        }
    }
    *chunk = best_per * attn_sm100::DEC_TK;
    *nsplit = (W + *chunk - 1) / *chunk;
}

int check_decode_args(int B, int H, int Hkv, int T, int W, int window, int d, float scale)
{
    if (B <= 0 || H <= 0 || Hkv <= 0 || T <= 0 || W <= 0 || d <= 0) return ATTN_ERR_INVALID;
    if (H % Hkv != 0) return ATTN_ERR_INVALID;
    // every position of every token's window must still be in the cache
    if (window < 0 || static_cast<int64_t>(window) + T > W) return ATTN_ERR_INVALID;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID;
    const int64_t bkv = static_cast<int64_t>(B) * Hkv;
    if (static_cast<int64_t>(B) * H * T > INT_MAX || bkv > 65535) return ATTN_ERR_UNSUPPORTED;
    if (bkv * W > INT64_MAX / (4 * static_cast<int64_t>(d))) return ATTN_ERR_INVALID;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    // the G query heads of a group times the T tokens fill one 16-wide MMA
    if (static_cast<int64_t>(H / Hkv) * T > attn_sm100::DEC_N) return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

size_t decode_workspace(int B, int H, int Hkv, int T, int W, int d)
{
    int nsplit = 0, chunk = 0;
    choose_splits(static_cast<int64_t>(B) * Hkv, W, &nsplit, &chunk);
    return static_cast<size_t>(nsplit) * B * H * T * (d + 2) * 4;
}

// Cache [bkv, W, d] bf16 as a 3-D tensor (d fastest), boxes of 64 columns x
// 128 slots x 1, 128-byte swizzle; slots past W read as zero.
bool encode_cache(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *m, const void *ptr, int64_t bkv,
                  int64_t W, int64_t d)
{
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(W),
                          static_cast<cuuint64_t>(bkv)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(W * d * 2)};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(attn_sm100::BOX_COLS),
                         static_cast<cuuint32_t>(attn_sm100::DEC_TK), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NC>
int launch_decode(const void *q, const void *kc, const void *vc, const int *pos, void *o, float *lse,
                  float *part, int B, int H, int Hkv, int T, int W, int window, float scale, cudaStream_t stream,
                  int dev, int *status)
{
    using Cfg = attn_sm100::DecCfg<D, NC>;
    auto enc = encoder();
    if (!enc) return ATTN_ERR_CUDA;
    const int64_t bkv = static_cast<int64_t>(B) * Hkv;
    CUtensorMap mk, mv;
    if (!encode_cache(enc, &mk, kc, bkv, W, D) || !encode_cache(enc, &mv, vc, bkv, W, D)) return ATTN_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        bool &set = g_dec_set[dev][D == 128 ? 1 : 0][NC == 1 ? 0 : NC == 2 ? 1 : NC == 4 ? 2 : NC == 8 ? 3 : 4];
        if (!set) {
            if (cudaFuncSetAttribute(attn_sm100::attn_decode_kernel<D, NC>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess)
                return ATTN_ERR_CUDA;
            set = true;
        }
    }
    attn_sm100::DecodeParams p;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.pos = pos;
    p.part = part;
    p.status = status;
    p.H = H;
    p.Hkv = Hkv;
    p.W = W;
    p.T = T;
    p.window = window;
    choose_splits(bkv, W, &p.nsplit, &p.chunk);
    p.scale_log2 = scale * 1.4426950408889634f;
    const dim3 grid(static_cast<unsigned>(p.nsplit), static_cast<unsigned>(bkv));
    attn_sm100::attn_decode_kernel<D, NC><<<grid, attn_sm100::DEC_THREADS, Cfg::SMEM_BYTES, stream>>>(mk, mv, p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    const int rows = B * H * T;
    attn_sm100::attn_decode_combine_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
        part, static_cast<__nv_bfloat16 *>(o), lse, rows, p.nsplit);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// The kernel instance whose column count NC is the G * T columns in use
// rounded up to a power of two.
template <int D>
int launch_decode_nc(const void *q, const void *kc, const void *vc, const int *pos, void *o, float *lse,
                     float *part, int B, int H, int Hkv, int T, int W, int window, float scale, cudaStream_t st,
                     int dev, int *status)
{
    const int gt = (H / Hkv) * T;
    if (gt <= 1) return launch_decode<D, 1>(q, kc, vc, pos, o, lse, part, B, H, Hkv, T, W, window, scale, st, dev, status);
    if (gt <= 2) return launch_decode<D, 2>(q, kc, vc, pos, o, lse, part, B, H, Hkv, T, W, window, scale, st, dev, status);
    if (gt <= 4) return launch_decode<D, 4>(q, kc, vc, pos, o, lse, part, B, H, Hkv, T, W, window, scale, st, dev, status);
    if (gt <= 8) return launch_decode<D, 8>(q, kc, vc, pos, o, lse, part, B, H, Hkv, T, W, window, scale, st, dev, status);
    return launch_decode<D, 16>(q, kc, vc, pos, o, lse, part, B, H, Hkv, T, W, window, scale, st, dev, status);
}

int decode_multi(const void *q, const void *k_cache, const void *v_cache, const int *pos, void *o, float *lse,
                 void *workspace, size_t workspace_bytes, int B, int H, int Hkv, int T, int W, int window, int d,
                 float scale, void *stream)
{
    if (!q || !k_cache || !v_cache || !pos || !o || !lse || !workspace) return ATTN_ERR_INVALID;
    const int rc = check_decode_args(B, H, Hkv, T, W, window, d, scale);
    if (rc != ATTN_OK) return rc;
    for (const void *ptr : {q, k_cache, v_cache, static_cast<const void *>(o), static_cast<const void *>(workspace)})
        if (!aligned(ptr, 16)) return ATTN_ERR_INVALID;
    if (!aligned(pos, 4) || !aligned(lse, 4)) return ATTN_ERR_INVALID;
    if (workspace_bytes < decode_workspace(B, H, Hkv, T, W, d)) return ATTN_ERR_INVALID;
    int dev = 0;
    if (current_device(&dev) != ATTN_OK) return ATTN_ERR_CUDA;
    int *status = status_word(dev);
    if (!status) return ATTN_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *part = static_cast<float *>(workspace);
    if (d == 64)
        return launch_decode_nc<64>(q, k_cache, v_cache, pos, o, lse, part, B, H, Hkv, T, W, window, scale, st, dev,
                                    status);
    return launch_decode_nc<128>(q, k_cache, v_cache, pos, o, lse, part, B, H, Hkv, T, W, window, scale, st, dev,
                                 status);
}

}  // namespace

extern "C" int64_t attn_decode_workspace_bytes(int B, int H, int Hkv, int W, int d)
{
    if (check_decode_args(B, H, Hkv, 1, W, W - 1, d, 1.f) != ATTN_OK) return -1;
    return static_cast<int64_t>(decode_workspace(B, H, Hkv, 1, W, d));
}

extern "C" int attn_decode(const void *q, const void *k_cache, const void *v_cache, const int *pos, void *o,
                           float *lse, void *workspace, size_t workspace_bytes, int B, int H, int Hkv, int W,
                           int d, float scale, void *stream)
{
    // one new token per sequence, window W - 1: every cached position
    return decode_multi(q, k_cache, v_cache, pos, o, lse, workspace, workspace_bytes, B, H, Hkv, 1, W, W - 1, d,
                        scale, stream);
}

extern "C" int64_t attn_decode_multi_workspace_bytes(int B, int H, int Hkv, int T, int W, int window, int d)
{
    if (check_decode_args(B, H, Hkv, T, W, window, d, 1.f) != ATTN_OK) return -1;
    return static_cast<int64_t>(decode_workspace(B, H, Hkv, T, W, d));
}

extern "C" int attn_decode_multi(const void *q, const void *k_cache, const void *v_cache, const int *pos, void *o,
                                 float *lse, void *workspace, size_t workspace_bytes, int B, int H, int Hkv, int T,
                                 int W, int window, int d, float scale, void *stream)
{
    return decode_multi(q, k_cache, v_cache, pos, o, lse, workspace, workspace_bytes, B, H, Hkv, T, W, window, d,
                        scale, stream);
}
