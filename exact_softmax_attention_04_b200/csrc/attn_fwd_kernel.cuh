// attn_fwd_kernel.cuh - exact softmax attention forward for sm_100a.
//
// One CTA computes one 128-row query tile Q_i of one (batch, head):
//   for each key/value tile j allowed by the mask:
//     S = Q_i K_j^T                       (tcgen05 MMA, smem x smem -> TMEM fp32)
//     online softmax on S, row by row     (running max m, running normaliser l)
//     O += P V_j                          (tcgen05 MMA, P from TMEM x V from smem)
//   O_i = O / l, LSE_i = m + ln l         (written once)
// This is the FlashAttention tile loop with the online softmax ("week17
// efficiency attention", FlashAttention section; "Efficient Transformers ...",
// "The online softmax trick"): the running output is kept unnormalised and
// divided once at the end, and only the current tile's scores live on chip.
//
// Roles (192 threads, 6 warps):
//   warps 0-3  softmax: thread r owns query row r (= TMEM lane r); reads S,
//              masks boundary tiles, updates (m, l), writes P (bf16) back into
//              TMEM over the S columns, rescales O when the max grew, and runs
//              the epilogue (O / l -> bf16 -> smem -> TMA store, LSE store).
//   warp 4     TMA producer (one elected lane): Q once, then K_j and V_j into
//              an NS-stage shared-memory ring.
//   warp 5     MMA issuer (one elected lane) and TMEM owner.
// TMEM columns: S/P double buffer at [0,128) and [128,256), O at [256, 256+D).
// S_{j+1} is computed while the softmax works on S_j; tcgen05 MMAs issued by
// one thread execute in order, so S_{j+2} never overwrites P_j before the
// P_j V_j MMA has read it.
//
// Every wait is bounded (about one second). On expiry the kernel records
// ATTN device status bit 1, tells the other roles to stop, waits (bounded) for
// its own copies and MMAs in flight, frees TMEM and returns.
#pragma once
#include <cuda_bf16.h>
#include <math_constants.h>

#include "sm100.cuh"

namespace attn_sm100 {

constexpr int BM = 128;  // query rows per tile (= TMEM lanes)
constexpr int BN = 128;  // keys per tile
constexpr int BOX_COLS = 64;                 // bf16 columns per 128-byte swizzle atom
constexpr int BOX_BYTES = BM * BOX_COLS * 2; // one [128 x 64] bf16 box: 16 KB
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;
constexpr uint64_t DRAIN_LIMIT_NS = 200000000ull;
constexpr int STATUS_WAIT_TIMEOUT = 1;
// The running max is replaced as soon as a tile raises it (threshold 0), so
// the largest P entry of a row is exactly 1.0 and its bf16 rounding never
// reaches O. A positive threshold (keeping a stale max, P up to 2^threshold)
// saves O rescales but puts up to 2^-9 relative error on the dominant term,
// which breaks the 2e-2 max-abs bar on O for peaked rows.
#ifndef ATTN_RESCALE_THRESHOLD
#define ATTN_RESCALE_THRESHOLD 0.0f
#endif
constexpr float RESCALE_THRESHOLD = ATTN_RESCALE_THRESHOLD;

struct FwdParams {
    float *lse;     // [B*H, n]
    int *status;    // device status word
    int n;
    int num_q_tiles;
    float scale_log2;  // scale * log2(e)
    int causal;
    int window;        // < 0: none
};

template <int D>
struct FwdCfg {
    static_assert(D == 64 || D == 128, "head size 64 or 128");
    static constexpr int NS = (D == 128) ? 3 : 4;       // K/V ring depth
    static constexpr int TILE_BYTES = BM * D * 2;        // 128 rows x D bf16
    static constexpr int BOXES = D / BOX_COLS;
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + TILE_BYTES;
    static constexpr int V_OFF = K_OFF + NS * TILE_BYTES;
    static constexpr int BAR_OFF = V_OFF + NS * TILE_BYTES;
    // q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], s_full[2],
    // p_full[2], o_done, drain
    static constexpr int NUM_BARS = 1 + 4 * NS + 2 + 2 + 1 + 1;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + 1 KB alignment slack
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t O_COL = 256;
    static constexpr int THREADS = 192;
};

struct Waiter {
    volatile int *abort_flag;
    int *status;

    // Bounded wait for the phase of `bar` with parity `parity` to complete.
    __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) const
    {
        if (mbar_try_wait(bar, parity)) return true;
        const uint64_t t0 = global_timer_ns();
        for (uint32_t it = 1;; ++it) {
            if (mbar_try_wait(bar, parity)) return true;
            if ((it & 15u) == 0) {
                if (*abort_flag) return false;
                if (global_timer_ns() - t0 > WAIT_LIMIT_NS) {
                    *abort_flag = 1;
                    atomicOr(status, STATUS_WAIT_TIMEOUT);
                    return false;
                }
            }
        }
    }

    // Wait used while shutting down: ignores the abort flag, shorter limit.
    __device__ __forceinline__ bool drain(uint32_t bar, uint32_t parity) const
    {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar, parity)) {
            if (global_timer_ns() - t0 > DRAIN_LIMIT_NS) {
                atomicOr(status, STATUS_WAIT_TIMEOUT);
                return false;
            }
        }
        return true;
    }
};

// Key tiles [jlo, jhi) that hold at least one key allowed for some row of the
// query tile starting at m0. Fully masked tiles are never visited.
__device__ __forceinline__ void key_tile_range(int m0, int n, int causal, int window, int &jlo,
                                               int &jhi)
{
    const int kend = causal ? min(n, m0 + BM) : n;           // exclusive
    const int kbeg = (window >= 0) ? max(0, m0 - window) : 0;
    jlo = kbeg / BN;
    jhi = (kend + BN - 1) / BN;
}

__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }
__device__ __forceinline__ uint32_t f2u(float x) { return __float_as_uint(x); }

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const FwdParams p)
{
    using C = FwdCfg<D>;
    constexpr int NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - raw);

    const uint32_t sQ = base + C::Q_OFF;
    const uint32_t bars = base + C::BAR_OFF;
    auto sK = [&](int s) { return base + C::K_OFF + s * C::TILE_BYTES; };
    auto sV = [&](int s) { return base + C::V_OFF + s * C::TILE_BYTES; };
    const uint32_t q_full = bars;
    auto k_full = [&](int s) { return bars + 8u * (1 + s); };
    auto k_empty = [&](int s) { return bars + 8u * (1 + NS + s); };
    auto v_full = [&](int s) { return bars + 8u * (1 + 2 * NS + s); };
    auto v_empty = [&](int s) { return bars + 8u * (1 + 3 * NS + s); };
    auto s_full = [&](int b) { return bars + 8u * (1 + 4 * NS + b); };
    auto p_full = [&](int b) { return bars + 8u * (3 + 4 * NS + b); };
    const uint32_t o_done = bars + 8u * (5 + 4 * NS);
    const uint32_t drain_bar = bars + 8u * (6 + 4 * NS);
    uint32_t *const tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + C::MISC_OFF);
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(base_ptr + C::MISC_OFF + 4);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    // Work tile: query tiles of one head are adjacent in blockIdx (K/V reuse in
    // L2); within a head the late (most expensive under a causal mask) tiles
    // start first.
    const int bh = blockIdx.x / p.num_q_tiles;
    const int qt = p.num_q_tiles - 1 - static_cast<int>(blockIdx.x % p.num_q_tiles);
    const int m0 = qt * BM;
    const int n = p.n;
    int jlo, jhi;
    key_tile_range(m0, n, p.causal, p.window, jlo, jhi);
    const int nt = jhi - jlo;  // >= 1: the diagonal tile always holds allowed keys

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(k_full(s), 1);
            mbar_init(k_empty(s), 1);
            mbar_init(v_full(s), 1);
            mbar_init(v_empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(s_full(b), 1);
            mbar_init(p_full(b), BM);
        }
        mbar_init(o_done, 1);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 4 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmO);
    }
    if (warp == 5) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Waiter wt{abort_flag, p.status};

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
            for (int b = 0; b < C::BOXES; ++b)
                tma_load_3d(sQ + b * BOX_BYTES, &tmQ, q_full, b * BOX_COLS, m0, bh);
            int kcount = 0, vcount = 0;
            bool ok = true;
            for (int t = 0; t < nt && ok; ++t) {
                const int s = t % NS;
                const uint32_t ph = (t / NS) & 1u;
                const int k0 = (jlo + t) * BN;
                if (t >= NS && !wt.wait(k_empty(s), ph ^ 1u)) { ok = false; break; }
                mbar_arrive_expect_tx(k_full(s), C::TILE_BYTES);
                for (int b = 0; b < C::BOXES; ++b)
                    tma_load_3d(sK(s) + b * BOX_BYTES, &tmK, k_full(s), b * BOX_COLS, k0, bh);
                ++kcount;
                if (t >= NS && !wt.wait(v_empty(s), ph ^ 1u)) { ok = false; break; }
                mbar_arrive_expect_tx(v_full(s), C::TILE_BYTES);
                for (int b = 0; b < C::BOXES; ++b)
                    tma_load_3d(sV(s) + b * BOX_BYTES, &tmV, v_full(s), b * BOX_COLS, k0, bh);
                ++vcount;
            }
            if (!ok) {
                // Let every copy issued into shared memory land before exiting.
                wt.drain(q_full, 0);
                for (int s = 0; s < NS; ++s) {
                    if (kcount > s) wt.drain(k_full(s), (((kcount - 1 - s) / NS)) & 1u);
                    if (vcount > s) wt.drain(v_full(s), (((vcount - 1 - s) / NS)) & 1u);
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, 0, 0);  // Q, K both K-major
            constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, 0, 1);   // P K-major, V MN-major
            bool ok = wt.wait(q_full, 0);
            tc_fence_after();
            for (int t = 0; ok && t <= nt; ++t) {
                if (t < nt) {
                    const int s = t % NS;
                    if (!wt.wait(k_full(s), (t / NS) & 1u)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d_s = tmem + static_cast<uint32_t>(t & 1) * BN;
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t off = (k / 4) * BOX_BYTES + (k % 4) * 32;
                        mma_bf16_ss(d_s, smem_desc_sw128(sQ + off, 16, 1024),
                                    smem_desc_sw128(sK(s) + off, 16, 1024), idesc_qk, k > 0);
                    }
                    mma_commit(k_empty(s));
                    mma_commit(s_full(t & 1));
                }
                if (t >= 1) {
                    const int u = t - 1;
                    const int s = u % NS;
                    if (!wt.wait(p_full(u & 1), (u >> 1) & 1u)) { ok = false; break; }
                    if (!wt.wait(v_full(s), (u / NS) & 1u)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_p = tmem + static_cast<uint32_t>(u & 1) * BN;
#pragma unroll
                    for (int k = 0; k < BN / 16; ++k) {
                        mma_bf16_ts(tmem + C::O_COL, a_p + k * 8,
                                    smem_desc_sw128(sV(s) + k * 16 * 128, BOX_BYTES, 1024), idesc_pv,
                                    (u > 0 || k > 0) ? 1u : 0u);
                    }
                    mma_commit(v_empty(s));
                    mma_commit(o_done);
                }
            }
            // Every MMA this thread issued must finish before TMEM is freed.
            mma_commit(drain_bar);
            wt.drain(drain_bar, 0);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int r = threadIdx.x;  // row in tile == TMEM lane
        const int row = m0 + r;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float sc = p.scale_log2;
        const int causal = p.causal, window = p.window;
        float mx = -CUDART_INF_F;  // running (possibly stale) max, log2 units
        float l = 0.f;             // running normaliser relative to mx
        bool ok = true;

        for (int t = 0; t < nt; ++t) {
            const int b = t & 1;
            ok = __all_sync(0xffffffffu, wt.wait(s_full(b), (t >> 1) & 1u));
            if (!ok) break;
            tc_fence_after();
            uint32_t s[BN];
#pragma unroll
            for (int c = 0; c < BN; c += 32)
                tmem_ld32(lane_base + b * BN + c, *reinterpret_cast<uint32_t(*)[32]>(&s[c]));

            const int k0 = (jlo + t) * BN;
            const bool need_mask = (k0 + BN > n) || (causal && k0 + BN - 1 > m0) ||
                                   (window >= 0 && k0 < m0 + BM - 1 - window);
            if (need_mask) {
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    const int key = k0 + c;
                    const bool allowed = key < n && (!causal || key <= row) &&
                                         (window < 0 || key >= row - window);
                    if (!allowed) s[c] = f2u(-CUDART_INF_F);
                }
            }
            float pm[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) pm[i] = u2f(s[i]);
#pragma unroll
            for (int c = 8; c < BN; ++c) pm[c & 7] = fmaxf(pm[c & 7], u2f(s[c]));
            const float tmax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                     fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
            const float mnew = tmax * sc;
            float alpha = 1.f;
            bool rescale = false;
            if (mnew > mx + RESCALE_THRESHOLD) {
                alpha = ex2_approx(mx - mnew);  // 0 when mx is -inf
                mx = mnew;
                rescale = true;
            }
            const float off = (mx == -CUDART_INF_F) ? 0.f : mx;  // no (-inf) - (-inf)
            float ps[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) ps[i] = 0.f;
#pragma unroll
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float e0 = ex2_approx(fmaf(u2f(s[c0 + 2 * i]), sc, -off));
                    const float e1 = ex2_approx(fmaf(u2f(s[c0 + 2 * i + 1]), sc, -off));
                    ps[(2 * i) & 7] += e0;
                    ps[(2 * i + 1) & 7] += e1;
                    pk[i] = pack_bf16x2(e0, e1);
                }
                tmem_st16(lane_base + b * BN + c0 / 2, pk);
            }
            const float tsum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
            l = l * alpha + tsum;

            if (t > 0) {
                // O holds P_{t-1} V_{t-1} once that MMA is done; rescale if needed.
                ok = __all_sync(0xffffffffu, wt.wait(o_done, (t - 1) & 1u));
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                    for (int c = 0; c < D; c += 32) {
                        uint32_t o[32];
                        tmem_ld32(lane_base + C::O_COL + c, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = f2u(u2f(o[i]) * alpha);
                        tmem_st32(lane_base + C::O_COL + c, o);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_full(b));
        }
        if (ok) ok = __all_sync(0xffffffffu, wt.wait(o_done, (nt - 1) & 1u));
        const bool all_ok = named_bar_and(1, BM, ok);
        if (all_ok) {
            tc_fence_after();
            // Epilogue: O / l -> bf16 -> swizzled smem (the Q buffer, free now)
            // -> TMA store; rows past n are clipped by the store.
            const float inv_l = 1.f / l;
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
                uint32_t o[32];
                tmem_ld32(lane_base + C::O_COL + c, o);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(u2f(o[2 * i]) * inv_l, u2f(o[2 * i + 1]) * inv_l);
                const uint32_t box = sQ + (c / BOX_COLS) * BOX_BYTES + r * 128;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t chunk = ((c % BOX_COLS) / 8 + q) ^ (r & 7);
                    st_shared_v4(box + chunk * 16, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(1, BM);
            if (threadIdx.x == 0) {
                for (int b = 0; b < C::BOXES; ++b)
                    tma_store_3d(&tmO, sQ + b * BOX_BYTES, b * BOX_COLS, m0, bh);
                tma_store_commit();
                tma_store_wait_read0();
            }
            if (row < n)
                p.lse[static_cast<size_t>(bh) * n + row] = (mx + __log2f(l)) * 0.69314718055994531f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace attn_sm100
