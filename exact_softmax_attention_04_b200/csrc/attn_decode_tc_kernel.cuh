// attn_decode_tc_kernel.cuh - the decode step for head size 128 on the
// tensor cores.
//
// Same contract, work split and partial-result layout as attn_decode_kernel
// (one CTA per split of the cached slots and (sequence, kv head); partial O,
// running max and sum merged by attn_decode_combine_kernel). The step reads
// every cached key and value once; on the CUDA cores it is limited by the
// instructions spent per cached byte (each key converted and multiplied once
// per query head). Here both contractions of a 128-slot tile are tcgen05
// MMAs, so a tile costs a few hundred instructions and the kernel streams at
// HBM speed:
//   S^T  = K_tile q^T     M = 128 slots, N = 16 (the G query heads of the
//                         group, zero rows up to 16), K = d; fp32 in TMEM
//                         with lane = slot;
//   O^T += V_tile^T P^T   M = d = 128, N = 16, K = 128 slots: the V tile as
//                         it lands from TMA is the MN-major A operand, P^T a
//                         16-row K-major operand written by the softmax.
// Roles (192 threads):
//   warp 0     TMA producer: K_0, V_0, K_1, V_1, ... through one 3-stage ring
//              of 32 KB tiles;
//   warp 1     TMEM owner and MMA issuer, order S(0), S(1), PV(0), S(2),
//              PV(1), ... so the next scores are ready when the softmax ends
//              a tile;
//   warps 2-5  softmax, one thread per slot (= TMEM lane): per query head the
//              tile max over 128 slots (shuffles, then the four warps through
//              shared memory), running max, per-thread partial sums, P^T into
//              shared memory (bf16), and the rescale of O^T in TMEM when a
//              head's max grows. They finish with O^T (lane = column of d).
// About 110 KB of shared memory and 64 TMEM columns: two CTAs per SM.
#pragma once
#include "attn_decode_kernel.cuh"

namespace attn_sm100 {

constexpr int DTC_TK = 128;       // slots per tile
constexpr int DTC_N = 16;         // MMA N: query heads of the group, zero-padded
constexpr int DTC_NST = 3;        // ring stages (each holds one K or one V tile)
constexpr int DTC_THREADS = 192;

template <int G>
struct DecTcCfg {
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "query heads per key/value head: 1, 2, 4 or 8");
    static constexpr int D = 128;
    static constexpr int BOX_BYTES_T = DTC_TK * 128;          // [128 slots x 64 cols] bf16
    static constexpr int TILE_BYTES = 2 * BOX_BYTES_T;        // one K or V tile
    static constexpr int OPB_BOX = DTC_N * 128;               // 16 rows x 64 elements, 128-byte swizzle
    static constexpr int OPB_BYTES = 2 * OPB_BOX;             // 16 rows x 128 elements
    static constexpr int RING_OFF = 0;
    static constexpr int Q_OFF = DTC_NST * TILE_BYTES;        // q, the B operand of S^T
    static constexpr int P_OFF = Q_OFF + OPB_BYTES;           // two P^T buffers
    static constexpr int RED_OFF = P_OFF + 2 * OPB_BYTES;     // fp32 [3][4 warps][8]
    static constexpr int BAR_OFF = RED_OFF + 3 * 4 * 8 * 4;
    // full[NST], empty[NST], s_full[2], s_free[2], p_full[2], pv_done[2], mma_drain
    static constexpr int NBAR = 2 * DTC_NST + 9;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;       // TMEM base (4 B), abort flag (4 B)
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;   // + slack to align the base to 1 KB
    static constexpr uint32_t TMEM_COLS = 64;
    static constexpr uint32_t S_COL = 0;                      // + 16 * buffer
    static constexpr uint32_t O_COL = 32;
    static_assert(Q_OFF % 1024 == 0 && P_OFF % 1024 == 0 && OPB_BYTES % 1024 == 0, "operand alignment");
    static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");
};

template <int G>
__global__ void __launch_bounds__(DTC_THREADS, 2)
    attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const DecodeParams p)
{
    using C = DecTcCfg<G>;
    constexpr int D = C::D;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - raw);
    auto ring = [&](int st) { return base + C::RING_OFF + st * C::TILE_BYTES; };
    const uint32_t sQ = base + C::Q_OFF;
    auto sP = [&](int pb) { return base + C::P_OFF + pb * C::OPB_BYTES; };
    float *const red = reinterpret_cast<float *>(base_ptr + C::RED_OFF);
    const uint32_t bars = base + C::BAR_OFF;
    auto full = [&](int st) { return bars + 8u * st; };
    auto empty = [&](int st) { return bars + 8u * (DTC_NST + st); };
    auto s_full = [&](int sb) { return bars + 8u * (2 * DTC_NST + sb); };
    auto s_free = [&](int sb) { return bars + 8u * (2 * DTC_NST + 2 + sb); };
    auto p_full = [&](int pb) { return bars + 8u * (2 * DTC_NST + 4 + pb); };
    auto pv_done = [&](int pb) { return bars + 8u * (2 * DTC_NST + 6 + pb); };
    const uint32_t mma_drain = bars + 8u * (2 * DTC_NST + 8);
    uint32_t *const tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + C::MISC_OFF);
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(base_ptr + C::MISC_OFF + 4);

    const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x / 32), 0);
    const int lane = static_cast<int>(threadIdx.x % 32);
    const int split = blockIdx.x;
    const int bkv = blockIdx.y;                 // b * Hkv + kv head
    const int b = bkv / p.Hkv;
    const int h0 = (bkv % p.Hkv) * G;           // first query head of the group
    const int pos = max(p.pos[b], 0);
    const int L = min(pos + 1, p.W);            // valid slots [0, L)
    const int s0 = split * p.chunk;
    const int s1 = min(s0 + p.chunk, L);
    const int ntiles = (s1 > s0) ? (s1 - s0 + DTC_TK - 1) / DTC_TK : 0;
    const size_t prow = static_cast<size_t>(b) * p.H + h0;  // partial row of head h0
    float *const part = p.part + static_cast<size_t>(split) * gridDim.y * G * (D + 2);

    if (ntiles == 0) {
        // no cached slot in this split: an empty partial (max -inf, sum 0)
        for (int i = threadIdx.x; i < G * (D + 2); i += DTC_THREADS) {
            const int g = i / (D + 2), c = i % (D + 2);
            part[(prow + g) * (D + 2) + c] = (c == D) ? -CUDART_INF_F : 0.f;
        }
        return;
    }

    if (threadIdx.x == 0) {
        for (int st = 0; st < DTC_NST; ++st) {
            mbar_init(full(st), 1);
            mbar_init(empty(st), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(s_full(i), 1);
            mbar_init(s_free(i), 4 * 32);
            mbar_init(p_full(i), 4 * 32);
            mbar_init(pv_done(i), 1);
        }
        mbar_init(mma_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // q of the group's G heads as a 16-row K-major operand (128-byte swizzle:
    // 16-byte chunk j of row g at chunk j ^ (g % 8)); rows >= G and both P^T
    // buffers zero (rows >= G of P^T stay zero for good).
    for (int i = threadIdx.x; i < DTC_N * (D / 8); i += DTC_THREADS) {
        const int g = i / (D / 8), j = i % (D / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (g < G)
            v = *reinterpret_cast<const uint4 *>(p.q + (static_cast<size_t>(b) * p.H + h0 + g) * D + 8 * j);
        const uint32_t addr = sQ + (j / 8) * C::OPB_BOX + g * 128 +
                              ((static_cast<uint32_t>(j % 8) ^ static_cast<uint32_t>(g & 7)) * 16);
        st_shared_v4(addr, v.x, v.y, v.z, v.w);
    }
    for (int i = threadIdx.x; i < 2 * C::OPB_BYTES / 16; i += DTC_THREADS)
        st_shared_v4(sP(0) + i * 16, 0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Waiter wt{abort_flag, p.status};

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        const uint32_t leader = elect_one();
        const int nitems = 2 * ntiles;  // item 2i: K_i, item 2i + 1: V_i
        int issued = 0;
        for (; issued < nitems; ++issued) {
            const int st = issued % DTC_NST;
            if (issued >= DTC_NST &&
                !__all_sync(0xffffffffu, wt.wait(empty(st), ((issued / DTC_NST) - 1) & 1u)))
                break;
            const int slot = s0 + (issued / 2) * DTC_TK;
            const CUtensorMap *map = (issued & 1) ? &tmV : &tmK;
            mbar_arrive_expect_tx_if(leader, full(st), C::TILE_BYTES);
#pragma unroll
            for (int bx = 0; bx < 2; ++bx)
                tma_load_3d_if(leader, ring(st) + bx * C::BOX_BYTES_T, map, full(st), bx * BOX_COLS, slot, bkv);
        }
        // copies still in flight must land before the CTA exits
        for (int st = 0; st < DTC_NST; ++st) {
            if (issued > st) {
                const int last = st + ((issued - 1 - st) / DTC_NST) * DTC_NST;
                wt.drain(full(st), (last / DTC_NST) & 1u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t leader = elect_one();
        constexpr uint32_t idesc_s = idesc_bf16_f32(DTC_TK, DTC_N, 0, 0);  // K, q both K-major
        constexpr uint32_t idesc_o = idesc_bf16_f32(D, DTC_N, 1, 0);       // V^T MN-major, P^T K-major
        const uint64_t qdesc = smem_desc_sw128(sQ, 16, 1024);
        // S(i) = K_i q^T into S buffer i % 2
        auto issue_s = [&](int i) -> bool {
            const int item = 2 * i, st = item % DTC_NST;
            if (!__all_sync(0xffffffffu, wt.wait(full(st), (item / DTC_NST) & 1u))) return false;
            // the softmax must have read S(i - 2) out of this buffer
            if (i >= 2 && !__all_sync(0xffffffffu, wt.wait(s_free(i % 2), ((i - 2) / 2) & 1u))) return false;
            tc_fence_after();
            const uint64_t kdesc = smem_desc_sw128(ring(st), 16, 1024);
            const uint32_t d_col = tmem + C::S_COL + DTC_N * (i % 2);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint64_t koff = static_cast<uint64_t>(((k / 4) * C::BOX_BYTES_T + (k % 4) * 32) >> 4);
                const uint64_t qoff = static_cast<uint64_t>(((k / 4) * C::OPB_BOX + (k % 4) * 32) >> 4);
                mma_bf16_ss_if(leader, d_col, kdesc + koff, qdesc + qoff, idesc_s, k > 0 ? 1u : 0u);
            }
            mma_commit_if(leader, s_full(i % 2));
            mma_commit_if(leader, empty(st));
            return true;
        };
        // O^T += V_i^T P_i^T
        auto issue_pv = [&](int i) -> bool {
            const int item = 2 * i + 1, st = item % DTC_NST;
            if (!__all_sync(0xffffffffu, wt.wait(full(st), (item / DTC_NST) & 1u))) return false;
            if (!__all_sync(0xffffffffu, wt.wait(p_full(i % 2), (i / 2) & 1u))) return false;
            tc_fence_after();
            const uint64_t vdesc = smem_desc_sw128(ring(st), C::BOX_BYTES_T, 1024);
            const uint64_t pdesc = smem_desc_sw128(sP(i % 2), 16, 1024);
#pragma unroll
            for (int k = 0; k < DTC_TK / 16; ++k) {
                const uint64_t poff = static_cast<uint64_t>(((k / 4) * C::OPB_BOX + (k % 4) * 32) >> 4);
                mma_bf16_ss_if(leader, tmem + C::O_COL, vdesc + static_cast<uint64_t>(k * 128), pdesc + poff,
                               idesc_o, (i > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit_if(leader, pv_done(i % 2));
            mma_commit_if(leader, empty(st));
            return true;
        };
        bool ok = issue_s(0);
        for (int i = 0; ok && i < ntiles; ++i) {
            if (i + 1 < ntiles) ok = issue_s(i + 1);
            if (ok) ok = issue_pv(i);
        }
        // every MMA this warp issued must finish before TMEM is freed
        mma_commit_if(leader, mma_drain);
        wt.drain(mma_drain, 0);
    } else {
        // ------------------------------------------------------------ softmax
        const int sw = warp % 4;                    // TMEM subpartition of this warp
        const int r = sw * 32 + lane;               // slot in the tile; column of d for O^T
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(sw * 32) << 16);
        const float sc = p.scale_log2;
        float m_run[G], l_part[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m_run[g] = -CUDART_INF_F;
            l_part[g] = 0.f;
        }
        // Every tile the four warps agree (bar.red.and) before they exchange
        // maxima, so a wait that gives up in one warp ends the loop in all.
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const int sb = i % 2;
            bool okw = __all_sync(0xffffffffu, wt.wait(s_full(sb), (i / 2) & 1u));
            float s[G];
            if (okw) {
                tc_fence_after();
                uint32_t sv[8];
                tmem_ld8(lane_base + C::S_COL + DTC_N * sb, sv);
                tc_fence_before();
                mbar_arrive(s_free(sb));
                const bool valid = s0 + i * DTC_TK + r < s1;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    s[g] = valid ? __uint_as_float(sv[g]) * sc : -CUDART_INF_F;
                    float mx = s[g];
#pragma unroll
                    for (int o = 16; o >= 1; o /= 2) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    if (lane == 0) red[(sb * 4 + sw) * 8 + g] = mx;
                }
            }
            ok = named_bar_and(1, 4 * 32, okw);
            if (!ok) break;
            const int slot0 = s0 + i * DTC_TK;
            const bool valid = slot0 + r < s1;
            float alpha[G], pr[G];
            bool grew = false;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float tmax = fmaxf(fmaxf(red[(sb * 4 + 0) * 8 + g], red[(sb * 4 + 1) * 8 + g]),
                                         fmaxf(red[(sb * 4 + 2) * 8 + g], red[(sb * 4 + 3) * 8 + g]));
                const float m_new = fmaxf(m_run[g], tmax);  // finite: a tile's first slot is valid
                grew = grew || (m_new > m_run[g]);
                alpha[g] = ex2_approx(m_run[g] - m_new);    // 0 on the first tile
                pr[g] = ex2_approx(s[g] - m_new);           // 0 for slots past the cache
                l_part[g] = fmaf(l_part[g], alpha[g], pr[g]);
                m_run[g] = m_new;
            }
            // P^T buffer sb was last read by PV(i - 2)
            if (i >= 2) okw = __all_sync(0xffffffffu, wt.wait(pv_done(sb), ((i - 2) / 2) & 1u));
            // O^T must be rescaled when a head's max grew: it holds the tiles
            // before i once PV(i - 1) is done (the decision is the same in
            // every thread: all read the same maxima)
            if (okw && i > 0 && grew) {
                okw = __all_sync(0xffffffffu, wt.wait(pv_done((i - 1) % 2), ((i - 1) / 2) & 1u));
                if (okw) {
                    tc_fence_after();
                    uint32_t o[8];
                    tmem_ld8(lane_base + C::O_COL, o);
#pragma unroll
                    for (int g = 0; g < G; ++g) o[g] = __float_as_uint(__uint_as_float(o[g]) * alpha[g]);
                    tmem_st8(lane_base + C::O_COL, o);
                    tmem_wait_st();
                }
            }
            // Slots in [L, W) hold whatever the caller left there; their P is
            // 0, but 0 * NaN would still reach O, so their V rows are zeroed
            // (slots >= W already read as zero).
            if (okw && slot0 + DTC_TK > s1 && s1 < p.W) {
                const int item = 2 * i + 1, st = item % DTC_NST;
                okw = __all_sync(0xffffffffu, wt.wait(full(st), (item / DTC_NST) & 1u));
                if (okw && !valid && slot0 + r < p.W) {
#pragma unroll
                    for (int bx = 0; bx < 2; ++bx)
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            st_shared_v4(ring(st) + bx * C::BOX_BYTES_T + r * 128 + c * 16, 0u, 0u, 0u, 0u);
                }
            }
            if (okw) {
                // P^T: row g (head), column r (slot)
                const uint32_t col = sP(sb) + (r / 64) * C::OPB_BOX +
                                     ((static_cast<uint32_t>((r % 64) / 8)) * 16) + (r % 8) * 2;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const uint32_t addr = (col + g * 128) ^ (static_cast<uint32_t>(g & 7) << 4);
                    const unsigned short h = __bfloat16_as_ushort(__float2bfloat16_rn(pr[g]));
                    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(h) : "memory");
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(p_full(sb));
            }
            ok = okw;
        }
        // the four warps agree on how the loop ended
        ok = named_bar_and(1, 4 * 32, ok);
        bool okw = ok;
        if (ok) {
            const int last = ntiles - 1;
            okw = __all_sync(0xffffffffu, wt.wait(pv_done(last % 2), (last / 2) & 1u));
            if (okw) {
                tc_fence_after();
                uint32_t o[8];
                tmem_ld8(lane_base + C::O_COL, o);
                // O^T lane r = column r of d, column g = head g
#pragma unroll
                for (int g = 0; g < G; ++g) part[(prow + g) * (D + 2) + r] = __uint_as_float(o[g]);
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float sum = l_part[g];
#pragma unroll
                for (int o = 16; o >= 1; o /= 2) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (lane == 0) red[(2 * 4 + sw) * 8 + g] = sum;
            }
        }
        ok = named_bar_and(1, 4 * 32, okw);
        if (ok) {
            // this split's max and sum of head g, written by thread g (every
            // thread holds the same running maxima)
#pragma unroll
            for (int g = 0; g < G; ++g) {
                if (r == g) {
                    const float l = (red[(2 * 4 + 0) * 8 + g] + red[(2 * 4 + 1) * 8 + g]) +
                                    (red[(2 * 4 + 2) * 8 + g] + red[(2 * 4 + 3) * 8 + g]);
                    part[(prow + g) * (D + 2) + D] = m_run[g];
                    part[(prow + g) * (D + 2) + D + 1] = l;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace attn_sm100
