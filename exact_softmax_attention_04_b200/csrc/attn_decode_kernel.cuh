// attn_decode_kernel.cuh - one decode step against rolling key/value caches.
//
// Each sequence b has T new query tokens (T = 1 for plain decoding, a few for
// speculative or chunked steps) at positions t_u = pos[b] - T + 1 + u; keys
// and values sit in a W-slot rolling cache, position p in slot p mod W, so
// once the new tokens are written the cache holds positions
// max(0, pos - W + 1) .. pos (the rolling buffer of the worked example on
// "Beyond attention", section "For engineers -- Show the maths": a
// 4,096-position cache serving n = 32,768). Token u attends to the positions
// max(0, t_u - w) .. t_u of its causal window w (w + T <= W keeps all of them
// in the cache). Softmax is invariant to the order of its terms, so the
// kernel walks the cached slots [0, L), L = min(pos + 1, W), in slot order and
// masks, per token, the slots whose position lies outside its window.
// Query head h reads key/value head h / G, G = H / Hkv (grouped-query
// attention, "week17 efficiency attention", MQA / GQA section). The G query
// heads of a group times the T tokens give the G*T <= 16 columns of the
// MMAs below (column c = g * T + u).
//
// The step reads every cached key and value once for 4*d FLOPs per (query
// head, key): it is bound by HBM bandwidth, and what decides how close it
// gets is the instruction count per cached byte. Both contractions of a
// 128-slot tile are therefore tcgen05 MMAs (a tile costs a few hundred
// instructions; on the CUDA cores every key is converted and multiplied once
// per query head):
//   S^T  = K_tile q^T     M = 128 slots, N = 16 (the G*T query rows of the
//                         group, zero rows up to 16), K = d; fp32 in TMEM
//                         with lane = slot;
//   O^T += V_tile^T P^T   M = d, N = 16, K = 128 slots: the V tile as it
//                         lands from TMA is the MN-major A operand, P^T a
//                         16-row K-major operand written by the softmax. At
//                         d = 64 the accumulator has M = 64 rows, which TMEM
//                         holds as 16 lanes of each 32-lane quarter (row
//                         16 q + i in lane 32 q + i).
//   attn_decode_kernel: one CTA per (split of the slots, batch * kv head),
//     192 threads:
//     warp 0     TMA producer: K_0, V_0, K_1, V_1, ... through one ring of
//                96 KB (3 stages of 32 KB tiles at d = 128, 6 of 16 KB at 64);
//     warp 1     TMEM owner and MMA issuer, order S(0), S(1), PV(0), S(2),
//                PV(1), ... so the next scores are ready when the softmax
//                ends a tile;
//     warps 2-5  softmax, one thread per slot (= TMEM lane): per column
//                the window mask of the slot's position, the tile max over
//                128 slots (shuffles, then the four warps through shared
//                memory), running max, per-thread partial sums, P^T into
//                shared memory (bf16), and the rescale of O^T in TMEM when a
//                column's max grows. They finish with O^T.
//     The CTA writes its unnormalised partial O, running max and sum. About
//     110 KB of shared memory and 64 TMEM columns: two CTAs per SM.
//   attn_decode_combine_kernel: merges the splits of every (b, h, token)
//     with the log-sum-exp rule and writes O (bf16) and LSE.
#pragma once
#include "attn_fwd_kernel.cuh"

namespace attn_sm100 {

struct DecodeParams {
    const __nv_bfloat16 *q;  // [B, H, T, D]
    const int *pos;          // [B], device: position of each sequence's last new token
    float *part;             // [nsplit][B*H*T][D + 2]: unnormalised O, max (log2 units), sum
    int *status;
    int H, Hkv, W;
    int T;                   // new tokens per sequence (G * T <= NC)
    int window;              // causal window w of every token (w + T <= W)
    int nsplit;
    int chunk;               // slots per split, a multiple of DEC_TK
    float scale_log2;        // scale * log2(e)
};

constexpr int DEC_TK = 128;       // slots per tile
constexpr int DEC_N = 16;         // MMA N: the G*T query rows of a group, zero-padded
constexpr int DEC_THREADS = 192;

// NC: columns the softmax handles, G*T rounded up to a power of two <= 16.
template <int D, int NC>
struct DecCfg {
    static_assert(D == 64 || D == 128, "head size 64 or 128");
    static_assert(NC == 1 || NC == 2 || NC == 4 || NC == 8 || NC == 16, "1, 2, 4, 8 or 16 columns");
    static constexpr int BOXES = D / BOX_COLS;                // 64-column boxes per row
    static constexpr int BOX_BYTES_T = DEC_TK * 128;          // [128 slots x 64 cols] bf16
    static constexpr int TILE_BYTES = BOXES * BOX_BYTES_T;    // one K or V tile
    static constexpr int NST = 3 * 128 / D;                   // ring stages (each one K or one V tile)
    static constexpr int OPB_BOX = DEC_N * 128;               // 16 rows x 64 elements, 128-byte swizzle
    static constexpr int OPB_BYTES = 2 * OPB_BOX;             // 16 rows x 128 elements (P^T)
    static constexpr int Q_BYTES = BOXES * OPB_BOX;           // 16 rows x D elements (q)
    static constexpr int RING_OFF = 0;
    static constexpr int Q_OFF = NST * TILE_BYTES;            // q, the B operand of S^T
    static constexpr int P_OFF = Q_OFF + Q_BYTES;             // two P^T buffers
    static constexpr int RED_OFF = P_OFF + 2 * OPB_BYTES;     // fp32 [3][4 warps][NC]
    static constexpr int BAR_OFF = RED_OFF + 3 * 4 * 16 * 4;
    // full[NST], empty[NST], s_full[2], s_free[2], p_full[2], pv_done[2], mma_drain
    static constexpr int NBAR = 2 * NST + 9;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;       // TMEM base (4 B), abort flag (4 B)
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;   // + slack to align the base to 1 KB
    static constexpr uint32_t TMEM_COLS = 64;
    static constexpr uint32_t S_COL = 0;                      // + 16 * buffer
    static constexpr uint32_t O_COL = 32;
    static_assert(Q_OFF % 1024 == 0 && P_OFF % 1024 == 0 && OPB_BYTES % 1024 == 0, "operand alignment");
    static_assert(NST * TILE_BYTES == 3 * 32768, "ring of 96 KB");
    static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");
};

// TMEM load of the first NC columns of a 32-lane quarter (8 at least).
template <int NC>
__device__ __forceinline__ void dec_tmem_ld(uint32_t taddr, uint32_t (&r)[NC < 8 ? 8 : NC])
{
    if constexpr (NC <= 8) {
        tmem_ld8(taddr, r);
    } else {
        uint32_t a[8], b[8];
        tmem_ld8(taddr, a);
        tmem_ld8(taddr + 8, b);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            r[i] = a[i];
            r[8 + i] = b[i];
        }
    }
}

template <int NC>
__device__ __forceinline__ void dec_tmem_st(uint32_t taddr, const uint32_t (&r)[NC < 8 ? 8 : NC])
{
    if constexpr (NC <= 8) {
        tmem_st8(taddr, r);
    } else {
        uint32_t a[8], b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            a[i] = r[i];
            b[i] = r[8 + i];
        }
        tmem_st8(taddr, a);
        tmem_st8(taddr + 8, b);
    }
}

template <int D, int NC>
__global__ void __launch_bounds__(DEC_THREADS, 2)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const DecodeParams p)
{
    using C = DecCfg<D, NC>;
    constexpr int NR = NC < 8 ? 8 : NC;  // TMEM columns read per load
    constexpr int NST = C::NST;
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
    auto empty = [&](int st) { return bars + 8u * (NST + st); };
    auto s_full = [&](int sb) { return bars + 8u * (2 * NST + sb); };
    auto s_free = [&](int sb) { return bars + 8u * (2 * NST + 2 + sb); };
    auto p_full = [&](int pb) { return bars + 8u * (2 * NST + 4 + pb); };
    auto pv_done = [&](int pb) { return bars + 8u * (2 * NST + 6 + pb); };
    const uint32_t mma_drain = bars + 8u * (2 * NST + 8);
    uint32_t *const tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + C::MISC_OFF);
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(base_ptr + C::MISC_OFF + 4);

    const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x / 32), 0);
    const int lane = static_cast<int>(threadIdx.x % 32);
    const int split = blockIdx.x;
    const int bkv = blockIdx.y;                 // b * Hkv + kv head
    const int G = p.H / p.Hkv;
    const int T = p.T;
    const int GT = G * T;                       // columns in use (<= NC)
    const int b = bkv / p.Hkv;
    const int h0 = (bkv % p.Hkv) * G;           // first query head of the group
    const int pos = max(p.pos[b], T - 1);       // position of the last new token
    const int L = min(pos + 1, p.W);            // cached slots [0, L)
    const int s0 = split * p.chunk;
    const int s1 = min(s0 + p.chunk, L);
    const int ntiles = (s1 > s0) ? (s1 - s0 + DEC_TK - 1) / DEC_TK : 0;
    // q and partial rows of column c = g * T + u: (b * H + h0 + g) * T + u
    const size_t prow = (static_cast<size_t>(b) * p.H + h0) * T;
    float *const part = p.part + static_cast<size_t>(split) * gridDim.y * GT * (D + 2);

    if (ntiles == 0) {
        // no cached slot in this split: an empty partial (max -inf, sum 0)
        for (int i = threadIdx.x; i < GT * (D + 2); i += DEC_THREADS) {
            const int c = i / (D + 2), e = i % (D + 2);
            part[(prow + c) * (D + 2) + e] = (e == D) ? -CUDART_INF_F : 0.f;
        }
        return;
    }

    if (threadIdx.x == 0) {
        for (int st = 0; st < NST; ++st) {
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
    // q of the group's G*T rows as a 16-row K-major operand (128-byte
    // swizzle: 16-byte chunk j of row c at chunk j ^ (c % 8)); rows >= G*T and
    // both P^T buffers zero (rows >= NC of P^T stay zero for good).
    for (int i = threadIdx.x; i < DEC_N * (D / 8); i += DEC_THREADS) {
        const int c = i / (D / 8), j = i % (D / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (c < GT) v = *reinterpret_cast<const uint4 *>(p.q + (prow + c) * D + 8 * j);
        const uint32_t addr = sQ + (j / 8) * C::OPB_BOX + c * 128 +
                              ((static_cast<uint32_t>(j % 8) ^ static_cast<uint32_t>(c & 7)) * 16);
        st_shared_v4(addr, v.x, v.y, v.z, v.w);
    }
    for (int i = threadIdx.x; i < 2 * C::OPB_BYTES / 16; i += DEC_THREADS)
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
            const int st = issued % NST;
            if (issued >= NST &&
                !__all_sync(0xffffffffu, wt.wait(empty(st), ((issued / NST) - 1) & 1u)))
                break;
            const int slot = s0 + (issued / 2) * DEC_TK;
            const CUtensorMap *map = (issued & 1) ? &tmV : &tmK;
#ifdef ATTN_FAULT_DEC_DROP_FIRST_K
            // Test hook (never defined in the library build): the first K
            // tile is never loaded, so every wait on it must expire and the
            // kernel must stop cleanly.
            if (issued == 0) continue;
#endif
            mbar_arrive_expect_tx_if(leader, full(st), C::TILE_BYTES);
#pragma unroll
            for (int bx = 0; bx < C::BOXES; ++bx)
                tma_load_3d_if(leader, ring(st) + bx * C::BOX_BYTES_T, map, full(st), bx * BOX_COLS, slot, bkv);
        }
        // copies still in flight must land before the CTA exits
        for (int st = 0; st < NST; ++st) {
            if (issued > st) {
                const int last = st + ((issued - 1 - st) / NST) * NST;
                wt.drain(full(st), (last / NST) & 1u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t leader = elect_one();
        constexpr uint32_t idesc_s = idesc_bf16_f32(DEC_TK, DEC_N, 0, 0);  // K, q both K-major
        constexpr uint32_t idesc_o = idesc_bf16_f32(D, DEC_N, 1, 0);       // V^T MN-major, P^T K-major
        const uint64_t qdesc = smem_desc_sw128(sQ, 16, 1024);
        // S(i) = K_i q^T into S buffer i % 2
        auto issue_s = [&](int i) -> bool {
            const int item = 2 * i, st = item % NST;
            if (!__all_sync(0xffffffffu, wt.wait(full(st), (item / NST) & 1u))) return false;
            // the softmax must have read S(i - 2) out of this buffer
            if (i >= 2 && !__all_sync(0xffffffffu, wt.wait(s_free(i % 2), ((i - 2) / 2) & 1u))) return false;
            tc_fence_after();
            const uint64_t kdesc = smem_desc_sw128(ring(st), 16, 1024);
            const uint32_t d_col = tmem + C::S_COL + DEC_N * (i % 2);
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
            const int item = 2 * i + 1, st = item % NST;
            if (!__all_sync(0xffffffffu, wt.wait(full(st), (item / NST) & 1u))) return false;
            if (!__all_sync(0xffffffffu, wt.wait(p_full(i % 2), (i / 2) & 1u))) return false;
            tc_fence_after();
            const uint64_t vdesc = smem_desc_sw128(ring(st), C::BOX_BYTES_T, 1024);
            const uint64_t pdesc = smem_desc_sw128(sP(i % 2), 16, 1024);
#pragma unroll
            for (int k = 0; k < DEC_TK / 16; ++k) {
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
        const int r = sw * 32 + lane;               // slot in the tile (= TMEM lane)
        // column of d that O^T holds in this thread's lane (d = 64: lanes
        // 16-31 of each quarter hold none)
        const int dcol = (D == 128) ? r : 16 * sw + lane;
        const bool has_dcol = (D == 128) || lane < 16;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(sw * 32) << 16);
        const float sc = p.scale_log2;
        // Window of each column's token: positions [lo, hi] (column c holds
        // token u = c % T at position pos - T + 1 + u); unused columns get an
        // empty interval.
        int lo_c[NC], hi_c[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int t_u = pos - T + 1 + c % T;
            hi_c[c] = (c < GT) ? t_u : -1;
            lo_c[c] = (c < GT) ? max(0, t_u - p.window) : 0;
        }
        float m_run[NC], l_part[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            m_run[c] = -CUDART_INF_F;
            l_part[c] = 0.f;
        }
        // Every tile the four warps agree (bar.red.and) before they exchange
        // maxima, so a wait that gives up in one warp ends the loop in all.
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const int sb = i % 2;
            const int slot = s0 + i * DEC_TK + r;
            const bool valid = slot < s1;
            // the position this slot holds (slots < L hold one)
            const int ppos = (pos < p.W) ? slot : pos - (pos - slot) % p.W;
            // Does any token attend to this slot? (A slot no token attends to
            // gets its V row zeroed below: its weight is 0, but 0 * NaN is not.)
            bool attended = false;
#pragma unroll
            for (int c = 0; c < NC; ++c) attended = attended || (valid && ppos >= lo_c[c] && ppos <= hi_c[c]);
            bool okw = __all_sync(0xffffffffu, wt.wait(s_full(sb), (i / 2) & 1u));
            float s[NC];
            if (okw) {
                tc_fence_after();
                uint32_t sv[NR];
                dec_tmem_ld<NC>(lane_base + C::S_COL + DEC_N * sb, sv);
                tc_fence_before();
                mbar_arrive(s_free(sb));
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    const bool allowed = valid && ppos >= lo_c[c] && ppos <= hi_c[c];
                    s[c] = allowed ? __uint_as_float(sv[c]) * sc : -CUDART_INF_F;
                    float mx = s[c];
#pragma unroll
                    for (int o = 16; o >= 1; o /= 2) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    if (lane == 0) red[(sb * 4 + sw) * 16 + c] = mx;
                }
            }
            // (ok carries a wait that gave up later in the previous tile)
            ok = named_bar_and(1, 4 * 32, okw && ok);
            if (!ok) break;
            float alpha[NC], pr[NC];
            bool grew = false;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const float tmax = fmaxf(fmaxf(red[(sb * 4 + 0) * 16 + c], red[(sb * 4 + 1) * 16 + c]),
                                         fmaxf(red[(sb * 4 + 2) * 16 + c], red[(sb * 4 + 3) * 16 + c]));
                const float m_new = fmaxf(m_run[c], tmax);
                grew = grew || (m_new > m_run[c]);
                // a column may have no allowed slot yet (-inf max): measure
                // from 0 then, so that no (-inf) - (-inf) arises
                const float m_ref = (m_new == -CUDART_INF_F) ? 0.f : m_new;
                alpha[c] = ex2_approx(m_run[c] - m_ref);    // 0 while the column was empty
                pr[c] = ex2_approx(s[c] - m_ref);           // 0 for masked slots
                l_part[c] = fmaf(l_part[c], alpha[c], pr[c]);
                m_run[c] = m_new;
            }
            // P^T buffer sb was last read by PV(i - 2)
            if (i >= 2) okw = __all_sync(0xffffffffu, wt.wait(pv_done(sb), ((i - 2) / 2) & 1u));
            // O^T must be rescaled when a column's max grew: it holds the
            // tiles before i once PV(i - 1) is done (the decision is the same
            // in every thread: all read the same maxima)
            if (okw && i > 0 && grew) {
                okw = __all_sync(0xffffffffu, wt.wait(pv_done((i - 1) % 2), ((i - 1) / 2) & 1u));
                if (okw) {
                    tc_fence_after();
                    uint32_t o[NR];
                    dec_tmem_ld<NC>(lane_base + C::O_COL, o);
#pragma unroll
                    for (int c = 0; c < NC; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha[c]);
                    dec_tmem_st<NC>(lane_base + C::O_COL, o);
                    tmem_wait_st();
                }
            }
            // Slots no token attends to: those in [L, W), which no position
            // has reached yet, and, with a window shorter than the cache, the
            // oldest cached ones. They may hold anything; their P is 0, but
            // 0 * NaN would still reach O, so their V rows are zeroed (slots
            // >= W already read as zero). Each warp decides for its own rows.
            const bool zero_row = !attended && slot < p.W;
            if (okw && __any_sync(0xffffffffu, zero_row)) {
                const int item = 2 * i + 1, st = item % NST;
                okw = __all_sync(0xffffffffu, wt.wait(full(st), (item / NST) & 1u));
                if (okw && zero_row) {
#pragma unroll
                    for (int bx = 0; bx < C::BOXES; ++bx)
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            st_shared_v4(ring(st) + bx * C::BOX_BYTES_T + r * 128 + e * 16, 0u, 0u, 0u, 0u);
                }
            }
            if (okw) {
                // P^T: row c (query row of the group), column r (slot)
                const uint32_t col = sP(sb) + (r / 64) * C::OPB_BOX +
                                     ((static_cast<uint32_t>((r % 64) / 8)) * 16) + (r % 8) * 2;
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    const uint32_t addr = (col + c * 128) ^ (static_cast<uint32_t>(c & 7) << 4);
                    const unsigned short h = __bfloat16_as_ushort(__float2bfloat16_rn(pr[c]));
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
                uint32_t o[NR];
                dec_tmem_ld<NC>(lane_base + C::O_COL, o);
                // O^T: this lane holds column dcol of d, TMEM column c = query row c
                if (has_dcol) {
#pragma unroll
                    for (int c = 0; c < NC; ++c)
                        if (c < GT) part[(prow + c) * (D + 2) + dcol] = __uint_as_float(o[c]);
                }
            }
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                float sum = l_part[c];
#pragma unroll
                for (int o = 16; o >= 1; o /= 2) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (lane == 0) red[(2 * 4 + sw) * 16 + c] = sum;
            }
        }
        ok = named_bar_and(1, 4 * 32, okw);
        if (ok) {
            // this split's max and sum of column c, written by thread c (every
            // thread holds the same running maxima)
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                if (r == c && c < GT) {
                    const float l = (red[(2 * 4 + 0) * 16 + c] + red[(2 * 4 + 1) * 16 + c]) +
                                    (red[(2 * 4 + 2) * 16 + c] + red[(2 * 4 + 3) * 16 + c]);
                    part[(prow + c) * (D + 2) + D] = m_run[c];
                    part[(prow + c) * (D + 2) + D + 1] = l;
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

// Merge the splits of each (b, h, token): M = max_s m_s, l = sum_s l_s 2^(m_s - M),
// O = sum_s O_s 2^(m_s - M) / l, LSE = (M + log2 l) ln 2. One warp per row.
template <int D>
__global__ void __launch_bounds__(256)
    attn_decode_combine_kernel(const float *__restrict__ part, __nv_bfloat16 *__restrict__ o,
                               float *__restrict__ lse, int rows, int nsplit)
{
    const int row = blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    float M = -CUDART_INF_F;
    for (int s = 0; s < nsplit; ++s) M = fmaxf(M, part[(static_cast<size_t>(s) * rows + row) * (D + 2) + D]);
    constexpr int PER = D / 32;
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    float l = 0.f;
    for (int s = 0; s < nsplit; ++s) {
        const float *ps = part + (static_cast<size_t>(s) * rows + row) * (D + 2);
        const float f = ex2_approx(ps[D] - M);  // 0 for an empty split
        l += ps[D + 1] * f;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] += ps[lane * PER + e] * f;
    }
    const float inv = 1.f / l;
#pragma unroll
    for (int e = 0; e < PER; ++e) o[static_cast<size_t>(row) * D + lane * PER + e] = __float2bfloat16_rn(acc[e] * inv);
    if (lane == 0) lse[row] = (M + __log2f(l)) * 0.69314718055994531f;
}

}  // namespace attn_sm100
