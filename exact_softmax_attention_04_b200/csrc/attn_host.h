// attn_host.h - host-side helpers shared by the library's translation units
// (forward and backward entry points): TMA descriptor encoding, the per-device
// status word, argument helpers. Internal: not part of the C ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

namespace attn_host {

constexpr int kMaxDevices = 64;

// Guards every lazily created per-device object of the library.
extern std::mutex g_mu;

bool aligned(const void *p, uintptr_t a);

// cuTensorMapEncodeTiled from the driver, looked up once; nullptr if absent.
PFN_cuTensorMapEncodeTiled_v12000 encoder();

// Device status word of `dev` (allocated and zeroed on first use). Kernels
// OR bits into it when a bounded wait expires; attn_sync_status reads and
// clears it. nullptr if the allocation fails.
int *status_word(int dev);

// [bh, n, d] bf16 viewed as a 3-D tensor (d fastest), boxes of 64 x 128 x 1,
// 128-byte swizzle; rows past n read as zero and are clipped on store.
bool encode_bhnd(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *m, const void *ptr, int64_t bh,
                 int64_t n, int64_t d);

// The window the kernels see: -1 (none) for window < 0 and for windows that
// reach every key (window >= n - 1, where the mask is the same without it),
// so kernel index arithmetic never meets a window wider than n.
int effective_window(int n, int window);

// The block size the kernels see: 0 (none) for block <= 0 and for blocks of
// n tokens or more (one block: the same keys as no block mask).
int effective_block(int n, int block);

// The calling thread's current device, checked against kMaxDevices.
int current_device(int *dev);

}  // namespace attn_host
