// attn_bwd_api.cu - host side of the backward pass: argument checks, workspace
// layout, TMA descriptors and the three launches (prep, dK/dV, dQ).
// Contracts in include/attn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>

#include "attn.h"
#include "attn_bwd_fused_kernel.cuh"
#include "attn_bwd_kernel.cuh"
#include "attn_host.h"

namespace {

using namespace attn_host;

bool g_bwd_set[kMaxDevices][2][2] = {};  // [device][d==128][general]
bool g_bwd_nomask_set[kMaxDevices][2] = {};  // kernels without mask code: [device][d==128]

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Head size 64 runs the fused kernel (dQ by reduce-adds into an fp32
// accumulator), head size 128 the split dK/dV and dQ kernels: each is the
// faster of the two designs measured at that head size.
bool fused_for(int d) { return d == 64; }

// Workspace layout: [dQ accumulator fp32 B*H*n*d (fused path only) |
// lse2 fp32 B*H*n_pad | delta fp32 B*H*n_pad], each part starting on a
// 256-byte boundary (n_pad = n rounded up to 128).
struct BwdWorkspace {
    size_t acc_bytes, stat_bytes, total;
};

BwdWorkspace workspace_layout(int64_t bh, int64_t n, int64_t d)
{
    const int64_t n_pad = (n + attn_sm100::BM - 1) / attn_sm100::BM * attn_sm100::BM;
    BwdWorkspace w;
    w.acc_bytes = fused_for(static_cast<int>(d)) ? round256(static_cast<size_t>(bh * n * d) * 4) : 0;
    w.stat_bytes = round256(static_cast<size_t>(bh * n_pad) * 4);
    w.total = w.acc_bytes + 2 * w.stat_bytes;
    return w;
}

// The fp32 dQ accumulator [bh, n, d] as a 3-D tensor for TMA reduce-adds:
// boxes of 32 columns (128 bytes) x 128 rows, 128-byte swizzle; rows past n
// are skipped.
bool encode_acc(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *m, float *ptr, int64_t bh, int64_t n,
                int64_t d)
{
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                          static_cast<cuuint64_t>(bh)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 4), static_cast<cuuint64_t>(n * d * 4)};
    cuuint32_t box[3] = {32, static_cast<cuuint32_t>(attn_sm100::BM), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int check_bwd_args(int B, int H, int n, int d, float scale, int causal)
{
    if (B <= 0 || H <= 0 || n <= 0 || d <= 0) return ATTN_ERR_INVALID;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID;
    const int64_t bh = static_cast<int64_t>(B) * H;
    if (bh > INT_MAX) return ATTN_ERR_INVALID;
    // the fp32 accumulator (4 bytes per element) must be addressable
    if (bh * n > INT64_MAX / (4 * static_cast<int64_t>(d) + 16)) return ATTN_ERR_INVALID;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (n > (1 << 30)) return ATTN_ERR_UNSUPPORTED;
    const int64_t tiles = bh * ((n + attn_sm100::BN - 1) / attn_sm100::BN);
    if (tiles > INT_MAX) return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

// The register split between warpgroups needs exactly the per-thread count it
// was computed for; refuse a build that differs (its raising warps would wait
// forever), and allow the kernel its dynamic shared memory.
template <typename Kernel>
int prepare_kernel(Kernel kernel, int smem_bytes, uint32_t regs_launch)
{
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return ATTN_ERR_CUDA;
    if (fa.numRegs != static_cast<int>(regs_launch)) return ATTN_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return ATTN_OK;
}

template <int D>
int launch_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
               const void *dout, void *dq, void *dk, void *dv, char *ws, int B, int H, int Hkv, int n,
               float scale, int causal, int window, int block, cudaStream_t stream, int dev, int *status)
{
    using KV = attn_sm100::BwdKVCfg<D>;
    using QC = attn_sm100::BwdQCfg<D>;
    auto enc = encoder();
    if (!enc) return ATTN_ERR_CUDA;
    const int64_t bh = static_cast<int64_t>(B) * H;
    const int64_t bhkv = static_cast<int64_t>(B) * Hkv;
    CUtensorMap mq, mk, mv, mdo, mdq, mdk, mdv;
    if (!encode_bhnd(enc, &mq, q, bh, n, D) || !encode_bhnd(enc, &mk, k, bhkv, n, D) ||
        !encode_bhnd(enc, &mv, v, bhkv, n, D) || !encode_bhnd(enc, &mdo, dout, bh, n, D) ||
        !encode_bhnd(enc, &mdq, dq, bh, n, D) || !encode_bhnd(enc, &mdk, dk, bhkv, n, D) ||
        !encode_bhnd(enc, &mdv, dv, bhkv, n, D))
        return ATTN_ERR_CUDA;
    const bool general = effective_block(n, block) > 0 || Hkv != H;
    // No mask and whole tiles: the builds without the mask test run it.
    const bool nomask = !general && !causal && effective_window(n, window) < 0 && n % attn_sm100::BN == 0;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        bool &set = nomask ? g_bwd_nomask_set[dev][D == 128 ? 1 : 0] : g_bwd_set[dev][D == 128 ? 1 : 0][general ? 1 : 0];
        if (!set) {
            int rc;
            if (general) {
                rc = prepare_kernel(attn_sm100::attn_bwd_dkdv_kernel<D, true, false>, KV::SMEM_BYTES, KV::REGS_LAUNCH);
                if (rc == ATTN_OK)
                    rc = prepare_kernel(attn_sm100::attn_bwd_dq_kernel<D, true, false>, QC::SMEM_BYTES, QC::REGS_LAUNCH);
            } else if (nomask) {
                rc = prepare_kernel(attn_sm100::attn_bwd_dkdv_kernel<D, false, true>, KV::SMEM_BYTES, KV::REGS_LAUNCH);
                if (rc == ATTN_OK)
                    rc = prepare_kernel(attn_sm100::attn_bwd_dq_kernel<D, false, true>, QC::SMEM_BYTES, QC::REGS_LAUNCH);
            } else {
                rc = prepare_kernel(attn_sm100::attn_bwd_dkdv_kernel<D, false, false>, KV::SMEM_BYTES, KV::REGS_LAUNCH);
                if (rc == ATTN_OK)
                    rc = prepare_kernel(attn_sm100::attn_bwd_dq_kernel<D, false, false>, QC::SMEM_BYTES, QC::REGS_LAUNCH);
            }
            if (rc != ATTN_OK) return rc;
            set = true;
        }
    }
    const BwdWorkspace w = workspace_layout(bh, n, D);
    float *lse2 = reinterpret_cast<float *>(ws + w.acc_bytes);
    float *delta = reinterpret_cast<float *>(ws + w.acc_bytes + w.stat_bytes);
    const int n_pad = (n + attn_sm100::BM - 1) / attn_sm100::BM * attn_sm100::BM;

    // 1. delta and lse2
    const int64_t prep_threads = bh * n_pad * (D / 8);
    const int64_t prep_blocks = (prep_threads + 255) / 256;
    if (prep_blocks > INT_MAX) return ATTN_ERR_UNSUPPORTED;
    attn_sm100::attn_bwd_prep_kernel<D><<<static_cast<unsigned>(prep_blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(dout), lse, lse2, delta,
        bh, n, n_pad);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;

    attn_sm100::BwdParams p;
    p.lse2 = lse2;
    p.delta = delta;
    p.status = status;
    p.heads = H;
    p.kv_heads = Hkv;
    p.n = n;
    p.n_pad = n_pad;
    p.num_k_tiles = (n + attn_sm100::BN - 1) / attn_sm100::BN;
    p.num_q_tiles = (n + attn_sm100::BM - 1) / attn_sm100::BM;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal;
    p.window = effective_window(n, window);
    p.block = effective_block(n, block);

    // 2. dK, dV: one CTA per key tile of each key/value head
    const unsigned kv_grid = static_cast<unsigned>(bhkv * p.num_k_tiles);
    if (general)
        attn_sm100::attn_bwd_dkdv_kernel<D, true, false><<<kv_grid, KV::THREADS, KV::SMEM_BYTES, stream>>>(
            mq, mk, mv, mdo, mdk, mdv, p);
    else if (nomask)
        attn_sm100::attn_bwd_dkdv_kernel<D, false, true><<<kv_grid, KV::THREADS, KV::SMEM_BYTES, stream>>>(
            mq, mk, mv, mdo, mdk, mdv, p);
    else
        attn_sm100::attn_bwd_dkdv_kernel<D, false, false><<<kv_grid, KV::THREADS, KV::SMEM_BYTES, stream>>>(
            mq, mk, mv, mdo, mdk, mdv, p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;

    // 3. dQ: one CTA per query tile
    const unsigned q_grid = static_cast<unsigned>(bh * p.num_q_tiles);
    if (general)
        attn_sm100::attn_bwd_dq_kernel<D, true, false><<<q_grid, QC::THREADS, QC::SMEM_BYTES, stream>>>(
            mq, mk, mv, mdo, mdq, p);
    else if (nomask)
        attn_sm100::attn_bwd_dq_kernel<D, false, true><<<q_grid, QC::THREADS, QC::SMEM_BYTES, stream>>>(
            mq, mk, mv, mdo, mdq, p);
    else
        attn_sm100::attn_bwd_dq_kernel<D, false, false><<<q_grid, QC::THREADS, QC::SMEM_BYTES, stream>>>(
            mq, mk, mv, mdo, mdq, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// The fused design: prep (delta, lse2, zeroed accumulator), one key-tile
// kernel, accumulator -> bf16 dQ.
template <int D>
int launch_bwd_fused(const void *q, const void *k, const void *v, const void *o, const float *lse,
                     const void *dout, void *dq, void *dk, void *dv, char *ws, int B, int H, int Hkv,
                     int n, float scale, int causal, int window, int block, cudaStream_t stream, int dev,
                     int *status)
{
    using Cfg = attn_sm100::FusedBwdCfg<D>;
    auto enc = encoder();
    if (!enc) return ATTN_ERR_CUDA;
    const int64_t bh = static_cast<int64_t>(B) * H;
    const int64_t bhkv = static_cast<int64_t>(B) * Hkv;
    CUtensorMap mq, mk, mv, mdo, mdk, mdv, macc;
    if (!encode_bhnd(enc, &mq, q, bh, n, D) || !encode_bhnd(enc, &mk, k, bhkv, n, D) ||
        !encode_bhnd(enc, &mv, v, bhkv, n, D) || !encode_bhnd(enc, &mdo, dout, bh, n, D) ||
        !encode_bhnd(enc, &mdk, dk, bhkv, n, D) || !encode_bhnd(enc, &mdv, dv, bhkv, n, D))
        return ATTN_ERR_CUDA;
    const bool general = effective_block(n, block) > 0 || Hkv != H;
    // No mask and whole tiles: no tile needs a mask, the build without the
    // mask test runs it.
    const bool nomask = !general && !causal && effective_window(n, window) < 0 && n % attn_sm100::BN == 0;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        bool &set = nomask ? g_bwd_nomask_set[dev][D == 128 ? 1 : 0] : g_bwd_set[dev][D == 128 ? 1 : 0][general ? 1 : 0];
        if (!set) {
            int rc;
            if (general)
                rc = prepare_kernel(attn_sm100::attn_bwd_fused_kernel<D, true, false>, Cfg::SMEM_BYTES,
                                    Cfg::REGS_LAUNCH);
            else if (nomask)
                rc = prepare_kernel(attn_sm100::attn_bwd_fused_kernel<D, false, true>, Cfg::SMEM_BYTES,
                                    Cfg::REGS_LAUNCH);
            else
                rc = prepare_kernel(attn_sm100::attn_bwd_fused_kernel<D, false, false>, Cfg::SMEM_BYTES,
                                    Cfg::REGS_LAUNCH);
            if (rc != ATTN_OK) return rc;
            set = true;
        }
    }
    const BwdWorkspace w = workspace_layout(bh, n, D);
    float *acc = reinterpret_cast<float *>(ws);
    if (!encode_acc(enc, &macc, acc, bh, n, D)) return ATTN_ERR_CUDA;
    float *lse2 = reinterpret_cast<float *>(ws + w.acc_bytes);
    float *delta = reinterpret_cast<float *>(ws + w.acc_bytes + w.stat_bytes);
    const int n_pad = (n + attn_sm100::BM - 1) / attn_sm100::BM * attn_sm100::BM;

    const int64_t prep_threads = bh * n_pad * (D / 8);
    const int64_t prep_blocks = (prep_threads + 255) / 256;
    if (prep_blocks > INT_MAX) return ATTN_ERR_UNSUPPORTED;
    attn_sm100::attn_bwd_fused_prep_kernel<D><<<static_cast<unsigned>(prep_blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(dout), lse, lse2, delta,
        acc, bh, n, n_pad);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;

    attn_sm100::FusedBwdParams p;
    p.dq_acc = acc;
    p.lse2 = lse2;
    p.delta = delta;
    p.status = status;
    p.heads = H;
    p.kv_heads = Hkv;
    p.n = n;
    p.n_pad = n_pad;
    p.num_k_tiles = (n + attn_sm100::BN - 1) / attn_sm100::BN;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal;
    p.window = effective_window(n, window);
    p.block = effective_block(n, block);
    const unsigned grid = static_cast<unsigned>(bhkv * p.num_k_tiles);
    if (general)
        attn_sm100::attn_bwd_fused_kernel<D, true, false><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(
            mq, mk, mv, mdo, mdk, mdv, macc, p);
    else if (nomask)
        attn_sm100::attn_bwd_fused_kernel<D, false, true><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(
            mq, mk, mv, mdo, mdk, mdv, macc, p);
    else
        attn_sm100::attn_bwd_fused_kernel<D, false, false><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(
            mq, mk, mv, mdo, mdk, mdv, macc, p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;

    const int64_t count8 = bh * n * D / 8;
    const int64_t conv_blocks = (count8 + 255) / 256;
    if (conv_blocks > INT_MAX) return ATTN_ERR_UNSUPPORTED;
    attn_sm100::attn_bwd_dq_convert_kernel<<<static_cast<unsigned>(conv_blocks), 256, 0, stream>>>(
        acc, static_cast<__nv_bfloat16 *>(dq), count8);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

extern "C" int64_t attn_bwd_workspace_bytes(int B, int H, int n, int d)
{
    if (check_bwd_args(B, H, n, d, 1.f, 0) != ATTN_OK) return -1;
    return static_cast<int64_t>(workspace_layout(static_cast<int64_t>(B) * H, n, d).total);
}

namespace {

int bwd_entry(const void *q, const void *k, const void *v, const void *o, const float *lse, const void *dout,
              void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes, int B, int H, int Hkv,
              int n, int d, float scale, int causal, int window, int block, void *stream)
{
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace) return ATTN_ERR_INVALID;
    if (Hkv <= 0 || H <= 0 || H % Hkv != 0) return ATTN_ERR_INVALID;
    const int rc = check_bwd_args(B, H, n, d, scale, causal);
    if (rc != ATTN_OK) return rc;
    for (const void *ptr : {q, k, v, o, dout, static_cast<const void *>(dq), static_cast<const void *>(dk),
                            static_cast<const void *>(dv), static_cast<const void *>(workspace)})
        if (!aligned(ptr, 16)) return ATTN_ERR_INVALID;
    if (!aligned(lse, 4)) return ATTN_ERR_INVALID;
    if (workspace_bytes < workspace_layout(static_cast<int64_t>(B) * H, n, d).total) return ATTN_ERR_INVALID;
    int dev = 0;
    if (current_device(&dev) != ATTN_OK) return ATTN_ERR_CUDA;
    int *status = status_word(dev);
    if (!status) return ATTN_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    if (fused_for(d))
        return launch_bwd_fused<64>(q, k, v, o, lse, dout, dq, dk, dv, ws, B, H, Hkv, n, scale, causal, window,
                                    block, st, dev, status);
    return launch_bwd<128>(q, k, v, o, lse, dout, dq, dk, dv, ws, B, H, Hkv, n, scale, causal, window, block,
                           st, dev, status);
}

}  // namespace

extern "C" int attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
                        const void *dout, void *dq, void *dk, void *dv, void *workspace,
                        size_t workspace_bytes, int B, int H, int n, int d, float scale, int causal,
                        int window, void *stream)
{
    return bwd_entry(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, H, n, d, scale, causal,
                     window, 0, stream);
}

extern "C" int attn_bwd_gqa(const void *q, const void *k, const void *v, const void *o, const float *lse,
                            const void *dout, void *dq, void *dk, void *dv, void *workspace,
                            size_t workspace_bytes, int B, int H, int Hkv, int n, int d, float scale, int causal,
                            int window, void *stream)
{
    return bwd_entry(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, n, d, scale,
                     causal, window, 0, stream);
}

extern "C" int attn_bwd_blocklocal(const void *q, const void *k, const void *v, const void *o, const float *lse,
                                   const void *dout, void *dq, void *dk, void *dv, void *workspace,
                                   size_t workspace_bytes, int B, int H, int Hkv, int n, int d, float scale,
                                   int causal, int block, void *stream)
{
    if (block <= 0) return ATTN_ERR_INVALID;
    return bwd_entry(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, n, d, scale,
                     causal, -1, block, stream);
}
