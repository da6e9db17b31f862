// attn_api.cu - host side of libattn_b200.so: argument checks, TMA descriptor
// encoding, launch, device status word, host-buffer entry point.
// The C declarations and their contracts are in include/attn.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "attn_fwd_kernel.cuh"
#include "attn_host.h"

namespace attn_host {

std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
bool g_encode_tried = false;
int *g_status[kMaxDevices] = {};

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encoder()
{
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode_tried) {
        g_encode_tried = true;
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    return g_encode;
}

int *status_word(int dev)
{
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status[dev]) {
        int *p = nullptr;
        if (cudaMalloc(&p, sizeof(int)) != cudaSuccess) return nullptr;
        if (cudaMemset(p, 0, sizeof(int)) != cudaSuccess) {
            cudaFree(p);
            return nullptr;
        }
        g_status[dev] = p;
    }
    return g_status[dev];
}

bool encode_bhnd(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *m, const void *ptr, int64_t bh,
                 int64_t n, int64_t d)
{
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                          static_cast<cuuint64_t>(bh)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(n * d * 2)};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(attn_sm100::BOX_COLS),
                         static_cast<cuuint32_t>(attn_sm100::BM), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int effective_window(int n, int window)
{
    return (window < 0 || window >= n - 1) ? -1 : window;
}

int effective_block(int n, int block)
{
    return (block <= 0 || block >= n) ? 0 : block;
}

int current_device(int *dev)
{
    if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return ATTN_ERR_CUDA;
    return ATTN_OK;
}

}  // namespace attn_host

namespace {

using namespace attn_host;

bool g_smem_set[kMaxDevices][2][2][2][2] = {};  // [device][d==128][block mask][persistent][no mask]
int g_num_sms[kMaxDevices] = {};

struct Staging {
    void *buf = nullptr;
    size_t cap = 0;
};
Staging g_staging[kMaxDevices];

// Side streams of attn_fwd_host, one per copy direction, so that one chunk
// of heads is copied in while another is computed and a third copied out.
#ifndef ATTN_HOST_CHUNKS
#define ATTN_HOST_CHUNKS 8
#endif
#ifndef ATTN_HOST_H2D_STREAMS
#define ATTN_HOST_H2D_STREAMS 1
#endif
constexpr int kHostChunks = ATTN_HOST_CHUNKS;
constexpr int kH2D = ATTN_HOST_H2D_STREAMS;  // copy-in streams, used by chunks in turn
struct HostPipe {
    cudaStream_t h2d[kH2D] = {}, d2h = nullptr;
    cudaEvent_t entry = nullptr, done = nullptr;
    cudaEvent_t in[kHostChunks] = {}, ran[kHostChunks] = {};
    bool ready = false;
};
HostPipe g_pipe[kMaxDevices];

// The current device's streams and events, created on first use (caller
// holds g_mu).
int host_pipe(int dev, HostPipe **out)
{
    HostPipe &hp = g_pipe[dev];
    if (!hp.ready) {
        // each handle is created once; after a failure, what exists is kept
        auto stream = [](cudaStream_t &h) {
            return h || cudaStreamCreateWithFlags(&h, cudaStreamNonBlocking) == cudaSuccess;
        };
        auto event = [](cudaEvent_t &e) {
            return e || cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
        };
        bool ok = stream(hp.d2h) && event(hp.entry) && event(hp.done);
        for (int i = 0; ok && i < kH2D; ++i) ok = stream(hp.h2d[i]);
        for (int c = 0; ok && c < kHostChunks; ++c) ok = event(hp.in[c]) && event(hp.ran[c]);
        if (!ok) return ATTN_ERR_CUDA;
        hp.ready = true;
    }
    *out = &hp;
    return ATTN_OK;
}

int check_args(const void *q, const void *k, const void *v, const void *o, const void *lse, int B,
               int H, int n, int d, float scale, int causal, int window, bool device_buffers,
               int Hkv = -1)
{
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID;
    if (B <= 0 || H <= 0 || n <= 0 || d <= 0) return ATTN_ERR_INVALID;
    if (Hkv != -1 && (Hkv <= 0 || H % Hkv != 0)) return ATTN_ERR_INVALID;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID;
    const int64_t bh = static_cast<int64_t>(B) * H;
    if (bh > INT_MAX) return ATTN_ERR_INVALID;
    if (bh * n > INT64_MAX / (2 * static_cast<int64_t>(d))) return ATTN_ERR_INVALID;
    if (device_buffers && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) ||
                           !aligned(o, 16) || !aligned(lse, 4)))
        return ATTN_ERR_INVALID;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (n > (1 << 30)) return ATTN_ERR_UNSUPPORTED;
    const int64_t tiles = bh * ((n + attn_sm100::BM - 1) / attn_sm100::BM);
    if (tiles > INT_MAX) return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

// Sets the kernel's launch attributes once per device and checks its
// register count against the split it was compiled for.
template <int D, bool BLOCKMASK, bool PERSIST, bool NOMASK>
int prepare_fwd(int dev)
{
    using Cfg = attn_sm100::FwdCfg<D>;
    std::lock_guard<std::mutex> lk(g_mu);
    bool &set = g_smem_set[dev][D == 128 ? 1 : 0][BLOCKMASK ? 1 : 0][PERSIST ? 1 : 0][NOMASK ? 1 : 0];
    if (set) return ATTN_OK;
    if (!g_num_sms[dev] &&
        (cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
         g_num_sms[dev] <= 0))
        return ATTN_ERR_CUDA;
    // The kernel moves registers between its warpgroups; that only works if it
    // is launched with exactly the per-thread register count the split was
    // computed for (else the raising warps wait forever). Refuse to launch a
    // build that differs.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, attn_sm100::attn_fwd_kernel<D, BLOCKMASK, PERSIST, NOMASK>) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (fa.numRegs != static_cast<int>(Cfg::REGS_LAUNCH)) return ATTN_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(attn_sm100::attn_fwd_kernel<D, BLOCKMASK, PERSIST, NOMASK>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::SMEM_BYTES) != cudaSuccess)
        return ATTN_ERR_CUDA;
    set = true;
    return ATTN_OK;
}

// Persistent schedule or one CTA per work item, and the persistent form's
// item order. Measured on one B200 over the target workloads (a sweep of
// n = 1024 ... 65536, d = 64 and 128, five masks, plus the configurations):
// - windows (and block masks) whose query tiles walk at most ~12 key tiles
//   (w = 256 and 1024, symmetric window 256): persistent, head-major order,
//   +3% to +29%; a CTA's set-up, Q load and epilogue are otherwise as long as
//   its key loop. w = 4096: one CTA per item (2% to 6% faster);
// - no mask: persistent only for short sequences (n <= 1536: +3% to +12%);
//   long rows: one CTA per item (persistent 2% to 7% slower);
// - causal without a window: persistent with pair-major items up to
//   n = 16384 (+3% to +18%: the hardware's CTA dispatch handles the unequal
//   causal items worse than the balanced snake), one CTA per item above
//   (2% to 9% faster at n >= 65536).
// ATTN_FWD_PERSIST_MAX_TILES (build time) moves the key-tile threshold; 0
// disables the persistent form in the automatic choice.
#ifndef ATTN_FWD_PERSIST_MAX_TILES
#define ATTN_FWD_PERSIST_MAX_TILES 12
#endif
std::atomic<int> g_schedule{ATTN_SCHEDULE_AUTO};

enum FwdSchedule { kPerItem = 0, kPersistHeadMajor = 1, kPersistPairMajor = 2 };

// window and block as the kernels see them (effective_window/_block).
FwdSchedule fwd_schedule(int n, int causal, int window, int block)
{
    const bool causal_only = causal && window < 0 && block <= 0;
    const FwdSchedule persist = causal_only ? kPersistPairMajor : kPersistHeadMajor;
    const int mode = g_schedule.load(std::memory_order_relaxed);
    if (mode == ATTN_SCHEDULE_PERSISTENT) return persist;
    if (mode == ATTN_SCHEDULE_PER_ITEM || ATTN_FWD_PERSIST_MAX_TILES <= 0) return kPerItem;
    if (causal_only) return n <= 16384 ? kPersistPairMajor : kPerItem;
    double keys;  // about the keys a query row attends to
    if (block > 0)
        keys = causal ? 1.5 * block : 2.0 * block;
    else if (window >= 0)
        keys = causal ? window : 2.0 * window;
    else
        keys = n;
    const double q_tiles = (n + attn_sm100::BM - 1) / attn_sm100::BM;
    const double tiles = std::min(q_tiles, keys / attn_sm100::BN + 2.0);
    return tiles <= ATTN_FWD_PERSIST_MAX_TILES ? kPersistHeadMajor : kPerItem;
}

template <int D>
int launch_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int n,
               float scale, int causal, int window, cudaStream_t stream, int dev, int *status,
               int Hkv = -1, int block = 0)
{
    using Cfg = attn_sm100::FwdCfg<D>;
    auto enc = encoder();
    if (!enc) return ATTN_ERR_CUDA;
    if (Hkv < 0) Hkv = H;
    const int64_t bh = static_cast<int64_t>(B) * H;
    const int64_t bhkv = static_cast<int64_t>(B) * Hkv;
    CUtensorMap mq, mk, mv, mo;
    if (!encode_bhnd(enc, &mq, q, bh, n, D) || !encode_bhnd(enc, &mk, k, bhkv, n, D) ||
        !encode_bhnd(enc, &mv, v, bhkv, n, D) || !encode_bhnd(enc, &mo, o, bh, n, D))
        return ATTN_ERR_CUDA;
    const bool blockmask = effective_block(n, block) > 0;
    attn_sm100::FwdParams p;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    p.status = status;
    p.heads = H;
    p.kv_heads = Hkv;
    p.n = n;
    p.num_q_tiles = (n + attn_sm100::BM - 1) / attn_sm100::BM;
    p.num_cta_tiles = (p.num_q_tiles + attn_sm100::QT - 1) / attn_sm100::QT;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal;
    p.window = effective_window(n, window);
    p.block = effective_block(n, block);
    p.num_work = static_cast<int>(bh * p.num_cta_tiles);
    const FwdSchedule sched = fwd_schedule(n, causal, p.window, p.block);
    const bool persist = sched != kPerItem;
    p.pair_major = sched == kPersistPairMajor ? 1 : 0;
    // No mask and whole key tiles: no tile is ever masked, so the build
    // without the mask code runs it.
    const bool nomask = !blockmask && !causal && p.window < 0 && n % attn_sm100::BN == 0;
    int prc = ATTN_OK;
    if (blockmask)
        prc = persist ? prepare_fwd<D, true, true, false>(dev) : prepare_fwd<D, true, false, false>(dev);
    else if (nomask)
        prc = persist ? prepare_fwd<D, false, true, true>(dev) : prepare_fwd<D, false, false, true>(dev);
    else
        prc = persist ? prepare_fwd<D, false, true, false>(dev) : prepare_fwd<D, false, false, false>(dev);
    if (prc != ATTN_OK) return prc;
    const unsigned grid = static_cast<unsigned>(persist ? std::min(p.num_work, g_num_sms[dev]) : p.num_work);
    using namespace attn_sm100;
    if (blockmask && persist)
        attn_fwd_kernel<D, true, true, false><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(mq, mk, mv, mo, p);
    else if (blockmask)
        attn_fwd_kernel<D, true, false, false><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(mq, mk, mv, mo, p);
    else if (nomask && persist)
        attn_fwd_kernel<D, false, true, true><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(mq, mk, mv, mo, p);
    else if (nomask)
        attn_fwd_kernel<D, false, false, true><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(mq, mk, mv, mo, p);
    else if (persist)
        attn_fwd_kernel<D, false, true, false><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(mq, mk, mv, mo, p);
    else
        attn_fwd_kernel<D, false, false, false><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(mq, mk, mv, mo, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

extern "C" int attn_fwd_schedule(int mode)
{
    if (mode != ATTN_SCHEDULE_AUTO && mode != ATTN_SCHEDULE_PER_ITEM && mode != ATTN_SCHEDULE_PERSISTENT)
        return -1;
    return g_schedule.exchange(mode);
}

extern "C" int attn_fwd_schedule_for(int n, int causal, int window, int block)
{
    if (n < 1) return -1;
    const int w = effective_window(n, window), b = effective_block(n, block);
    return fwd_schedule(n, causal ? 1 : 0, b > 0 ? -1 : w, b) == kPerItem ? ATTN_SCHEDULE_PER_ITEM
                                                                          : ATTN_SCHEDULE_PERSISTENT;
}

extern "C" int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                        int H, int n, int d, float scale, int causal, int window, void *stream)
{
    const int rc = check_args(q, k, v, o, lse, B, H, n, d, scale, causal, window, true);
    if (rc != ATTN_OK) return rc;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    int *status = status_word(dev);
    if (!status) return ATTN_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d == 64) return launch_fwd<64>(q, k, v, o, lse, B, H, n, scale, causal, window, st, dev, status);
    return launch_fwd<128>(q, k, v, o, lse, B, H, n, scale, causal, window, st, dev, status);
}

extern "C" int attn_fwd_gqa(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                            int H, int Hkv, int n, int d, float scale, int causal, int window,
                            void *stream)
{
    const int rc = check_args(q, k, v, o, lse, B, H, n, d, scale, causal, window, true, Hkv);
    if (rc != ATTN_OK) return rc;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    int *status = status_word(dev);
    if (!status) return ATTN_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d == 64)
        return launch_fwd<64>(q, k, v, o, lse, B, H, n, scale, causal, window, st, dev, status, Hkv);
    return launch_fwd<128>(q, k, v, o, lse, B, H, n, scale, causal, window, st, dev, status, Hkv);
}

extern "C" int attn_fwd_blocklocal(const void *q, const void *k, const void *v, void *o, float *lse,
                                   int B, int H, int Hkv, int n, int d, float scale, int causal, int block,
                                   void *stream)
{
    if (block <= 0) return ATTN_ERR_INVALID;
    const int rc = check_args(q, k, v, o, lse, B, H, n, d, scale, causal, -1, true, Hkv);
    if (rc != ATTN_OK) return rc;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    int *status = status_word(dev);
    if (!status) return ATTN_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d == 64)
        return launch_fwd<64>(q, k, v, o, lse, B, H, n, scale, causal, -1, st, dev, status, Hkv, block);
    return launch_fwd<128>(q, k, v, o, lse, B, H, n, scale, causal, -1, st, dev, status, Hkv, block);
}

extern "C" int attn_fwd_host(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                             int H, int n, int d, float scale, int causal, int window, void *stream)
{
    int rc = check_args(q, k, v, o, lse, B, H, n, d, scale, causal, window, false);
    if (rc != ATTN_OK) return rc;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    const size_t elems = static_cast<size_t>(B) * H * n * d;
    const size_t tb = (elems * 2 + 255) & ~static_cast<size_t>(255);
    const size_t lb = (static_cast<size_t>(B) * H * n * 4 + 255) & ~static_cast<size_t>(255);
    const size_t need = 4 * tb + lb;
    char *buf = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        Staging &s = g_staging[dev];
        if (s.cap < need) {
            if (s.buf) {
                cudaDeviceSynchronize();
                cudaFree(s.buf);
                s.buf = nullptr;
                s.cap = 0;
            }
            if (cudaMalloc(&s.buf, need) != cudaSuccess) {
                s.buf = nullptr;
                return ATTN_ERR_CUDA;
            }
            s.cap = need;
        }
        buf = static_cast<char *>(s.buf);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *dq = buf, *dk = buf + tb, *dv = buf + 2 * tb, *dout = buf + 3 * tb;
    float *dl = reinterpret_cast<float *>(buf + 4 * tb);
    const char *hq = static_cast<const char *>(q), *hk = static_cast<const char *>(k),
               *hv = static_cast<const char *>(v);
    char *ho = static_cast<char *>(o);

    // Heads are independent: cut them into up to kHostChunks chunks and
    // pipeline them (copy-in on one side stream, kernel on `stream`, copy-out
    // on the other), unless the problem is small enough for one pass.
    const int64_t bh = static_cast<int64_t>(B) * H;
    const size_t head_bytes = static_cast<size_t>(n) * d * 2;
    int chunks = (3 * elems * 2 >= (static_cast<size_t>(16) << 20)) ? kHostChunks : 1;
    if (chunks > bh) chunks = static_cast<int>(bh);
    const int64_t per = (bh + chunks - 1) / chunks;
    chunks = static_cast<int>((bh + per - 1) / per);
    if (chunks == 1) {
        if (cudaMemcpyAsync(dq, q, elems * 2, cudaMemcpyHostToDevice, st) != cudaSuccess ||
            cudaMemcpyAsync(dk, k, elems * 2, cudaMemcpyHostToDevice, st) != cudaSuccess ||
            cudaMemcpyAsync(dv, v, elems * 2, cudaMemcpyHostToDevice, st) != cudaSuccess)
            return ATTN_ERR_CUDA;
        rc = attn_fwd(dq, dk, dv, dout, dl, B, H, n, d, scale, causal, window, stream);
        if (rc != ATTN_OK) return rc;
        if (cudaMemcpyAsync(o, dout, elems * 2, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
            cudaMemcpyAsync(lse, dl, static_cast<size_t>(B) * H * n * 4, cudaMemcpyDeviceToHost, st) !=
                cudaSuccess)
            return ATTN_ERR_CUDA;
        return ATTN_OK;
    }
    HostPipe *hp = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        rc = host_pipe(dev, &hp);
    }
    if (rc != ATTN_OK) return rc;
    // Side-stream work starts after everything already on `stream` (the
    // staging buffers may still be in use by an earlier call), and `stream`
    // continues only once the last copy-out is done.
    if (cudaEventRecord(hp->entry, st) != cudaSuccess) return ATTN_ERR_CUDA;
    for (int i = 0; i < kH2D; ++i)
        if (cudaStreamWaitEvent(hp->h2d[i], hp->entry, 0) != cudaSuccess) return ATTN_ERR_CUDA;
    for (int c = 0; c < chunks; ++c) {
        const int64_t h0 = c * per;
        const int hc = static_cast<int>(bh - h0 < per ? bh - h0 : per);
        const size_t off = static_cast<size_t>(h0) * head_bytes, bytes = static_cast<size_t>(hc) * head_bytes;
        const size_t loff = static_cast<size_t>(h0) * n, lbytes = static_cast<size_t>(hc) * n * 4;
        cudaStream_t in_st = hp->h2d[c % kH2D];
        if (cudaMemcpyAsync(dq + off, hq + off, bytes, cudaMemcpyHostToDevice, in_st) != cudaSuccess ||
            cudaMemcpyAsync(dk + off, hk + off, bytes, cudaMemcpyHostToDevice, in_st) != cudaSuccess ||
            cudaMemcpyAsync(dv + off, hv + off, bytes, cudaMemcpyHostToDevice, in_st) != cudaSuccess ||
            cudaEventRecord(hp->in[c], in_st) != cudaSuccess || cudaStreamWaitEvent(st, hp->in[c], 0) != cudaSuccess)
            return ATTN_ERR_CUDA;
        rc = attn_fwd(dq + off, dk + off, dv + off, dout + off, dl + loff, 1, hc, n, d, scale, causal, window,
                      stream);
        if (rc != ATTN_OK) return rc;
        if (cudaEventRecord(hp->ran[c], st) != cudaSuccess || cudaStreamWaitEvent(hp->d2h, hp->ran[c], 0) != cudaSuccess ||
            cudaMemcpyAsync(ho + off, dout + off, bytes, cudaMemcpyDeviceToHost, hp->d2h) != cudaSuccess ||
            cudaMemcpyAsync(lse + loff, dl + loff, lbytes, cudaMemcpyDeviceToHost, hp->d2h) != cudaSuccess)
            return ATTN_ERR_CUDA;
    }
    if (cudaEventRecord(hp->done, hp->d2h) != cudaSuccess || cudaStreamWaitEvent(st, hp->done, 0) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return ATTN_OK;
}

extern "C" int attn_host_staging_release(void)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    Staging &s = g_staging[dev];
    if (s.buf) {
        if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
        if (cudaFree(s.buf) != cudaSuccess) return ATTN_ERR_CUDA;
        s.buf = nullptr;
        s.cap = 0;
    }
    return ATTN_OK;
}

extern "C" int attn_sync_status(void *stream)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    int *w = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        w = g_status[dev];
    }
    if (!w) return ATTN_OK;  // nothing launched on this device yet
    int h = 0;
    if (cudaMemcpy(&h, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
    if (h != 0) {
        if (cudaMemset(w, 0, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
        // bit 1: a bounded wait expired; any other bit: a kernel refused to run
        return (h & attn_sm100::STATUS_WAIT_TIMEOUT) ? ATTN_ERR_TIMEOUT : ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

extern "C" const char *attn_strerror(int status)
{
    switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration (head size must be 64 or 128, n at most 2^30)";
    case ATTN_ERR_CUDA: return "CUDA runtime or driver error";
    case ATTN_ERR_TIMEOUT: return "a kernel gave up on a bounded wait; outputs are undefined";
    case ATTN_ERR_TOO_LARGE: return "problem larger than the fixed scratch of attn_fwd_host_noalloc";
    default: return "unknown status";
    }
}

extern "C" int64_t attn_attended_pairs(int64_t n, int causal, int64_t window)
{
    if (n < 0) return -1;
    if (window >= 0 && !causal) {
        // symmetric window: sum_i min(n-1, i+w) - max(0, i-w) + 1
        if (window >= n - 1) return n * n;
        return n * (2 * window + 1) - window * (window + 1);
    }
    if (window >= 0 && window < n - 1)
        return (window + 1) * (window + 2) / 2 + (n - window - 1) * (window + 1);
    if (causal) return n * (n + 1) / 2;
    return n * n;
}

// ---------------------------------------------------------------------------
// attn_fwd_host_noalloc: the host-buffer entry point without any allocation.
// All of its device scratch sits in this file-scope array. In host code the
// name g_noalloc_scratch is only a host-side stand-in, never a device address:
// the address handed to copies and kernels comes from cudaGetSymbolAddress,
// resolved once per device with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

namespace {

void *g_noalloc_base[kMaxDevices] = {};

// Device address of g_noalloc_scratch on `dev` (the current device).
int noalloc_base(int dev, char **out)
{
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_noalloc_base[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ATTN_ERR_CUDA;
        g_noalloc_base[dev] = p;
    }
    *out = static_cast<char *>(g_noalloc_base[dev]);
    return ATTN_OK;
}

}  // namespace

extern "C" int attn_fwd_host_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                                     int B, int H, int n, int d, float scale, int causal, int window,
                                     void *stream)
{
    int rc = check_args(q, k, v, o, lse, B, H, n, d, scale, causal, window, false);
    if (rc != ATTN_OK) return rc;
    // Layout: [status word | q | k | v | o | lse], each part 256-byte aligned.
    const size_t elems = static_cast<size_t>(B) * H * n * d;
    const size_t tb = (elems * 2 + 255) & ~static_cast<size_t>(255);
    const size_t lbytes = static_cast<size_t>(B) * H * n * 4;
    const size_t lb = (lbytes + 255) & ~static_cast<size_t>(255);
    if (elems > ATTN_NOALLOC_SCRATCH_BYTES || 256 + 4 * tb + lb > ATTN_NOALLOC_SCRATCH_BYTES)
        return ATTN_ERR_TOO_LARGE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    char *base = nullptr;
    rc = noalloc_base(dev, &base);
    if (rc != ATTN_OK) return rc;
    int *status = reinterpret_cast<int *>(base);
    char *dq = base + 256, *dk = dq + tb, *dv = dk + tb, *dout = dv + tb;
    float *dl = reinterpret_cast<float *>(dout + tb);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The status word keeps the previous call's value: clear it first.
    if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess ||
        cudaMemcpyAsync(dq, q, elems * 2, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(dk, k, elems * 2, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(dv, v, elems * 2, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return ATTN_ERR_CUDA;
    rc = (d == 64) ? launch_fwd<64>(dq, dk, dv, dout, dl, B, H, n, scale, causal, window, st, dev, status)
                   : launch_fwd<128>(dq, dk, dv, dout, dl, B, H, n, scale, causal, window, st, dev, status);
    if (rc != ATTN_OK) return rc;
    if (cudaMemcpyAsync(o, dout, elems * 2, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemcpyAsync(lse, dl, lbytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return ATTN_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
    // The same reading of the status bits as attn_sync_status: bit 1 means a
    // bounded wait expired, any other bit that a kernel refused to run.
    if (h == 0) return ATTN_OK;
    return (h & attn_sm100::STATUS_WAIT_TIMEOUT) ? ATTN_ERR_TIMEOUT : ATTN_ERR_CUDA;
}
