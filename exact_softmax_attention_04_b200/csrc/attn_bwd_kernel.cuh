// attn_bwd_kernel.cuh - exact softmax attention backward pass for sm_100a.
//
// Gradients of L = sum(O * dO) with respect to Q, K, V, recomputing the
// attention weights from Q, K and the forward pass's LSE instead of storing
// them (the recompute that "Efficient Transformers: Sparse Attention, Linear
// Attention and FlashAttention", section "Family 3", attributes to
// FlashAttention's backward pass). With P_ij = exp(scale q_i.k_j - LSE_i) on
// allowed pairs and 0 elsewhere:
//   dV_j = sum_i P_ij dO_i
//   dP_ij = dO_i . v_j,  dS_ij = P_ij (dP_ij - delta_i),  delta_i = dO_i . O_i
//   dK_j = scale sum_i dS_ij q_i,  dQ_i = scale sum_j dS_ij k_j
// delta_i equals sum_j P_ij dP_ij because O_i = sum_j P_ij v_j.
//
// Three launches on one stream:
//   1. attn_bwd_prep_kernel: delta_i and LSE_i * log2(e) per row, padded to a
//      whole number of 128-row tiles per head.
//   2. attn_bwd_dkdv_kernel: one CTA per (batch * key/value head, 128-key
//      tile j). K_j, V_j stay in shared memory; the CTA walks the query tiles
//      i that attend to tile j, for every query head that reads this
//      key/value head (one for multi-head attention, H / H_kv for
//      grouped-query attention, whose dK and dV sum over the group), and
//      runs, per query tile, four tcgen05 MMAs:
//        S^T  = K_j Q_i^T   (smem x smem -> TMEM, 128 keys x 128 queries)
//        dP^T = V_j dO_i^T  (smem x smem -> TMEM)
//        dV  += P^T dO_i    (P^T in TMEM, over S^T's columns)
//        dK  += dS^T Q_i    (dS^T in TMEM, over dP^T's columns)
//      dV and dK accumulate in TMEM over the walk and are stored once.
//   3. attn_bwd_dq_kernel: one CTA per (batch * query head, 128-query tile
//      i), Q_i and dO_i held in TMEM as MMA operands; it walks the key tiles j
//      of the head's key/value head that tile i attends to and runs three MMAs
//      per key tile:
//        S  = Q_i K_j^T, dP = dO_i V_j^T   (TMEM x smem -> TMEM)
//        dQ += dS K_j                      (dS in TMEM, over dP's columns)
//      dQ accumulates in TMEM and is stored once.
// Computing dQ in a kernel of its own costs two more MMAs per tile pair (S
// and dP are recomputed) but needs no cross-CTA accumulation: adding each
// (key tile, query tile) contribution to a global fp32 dQ, by atomics or by
// TMA reduce-adds, was bound by the L2's reduction throughput (about
// 2.7 TB/s measured) at well under half the tensor-core rate.
//
// Roles of both main kernels (384 threads, 12 warps = 3 warpgroups):
//   warps 0-3, 4-7  "softmax": warpgroup h owns TMEM lanes 0-127 (thread r,
//                   lane r) and columns [64h, 64h+64) of the 128 x 128 tile.
//   warp 8          MMA issuer (one elected lane) and TMEM owner.
//   warp 9          TMA producer.
//   warps 10-11     idle.
// Registers: launched at 168 per thread; the softmax warpgroups raise to 232
// and the third drops to 40 (2*128*232 + 128*40 = 384*168).
//
// Every wait is bounded as in the forward kernel: on expiry the kernel sets
// bit 1 of the device status word, the other roles stop, copies and MMAs in
// flight are waited for (bounded), TMEM is freed and the kernel returns.
#pragma once
#include "attn_fwd_kernel.cuh"

namespace attn_sm100 {

// Of every 16 pairs of P entries a softmax thread computes, the first
// ATTN_BWD_EX2_EMU use the FMA-pipe polynomial for 2^x instead of the MUFU
// (masked entries are zeroed after the exponential, so the polynomial's
// range limit does not matter there).
#ifndef ATTN_BWD_EX2_EMU
#define ATTN_BWD_EX2_EMU 2
#endif
constexpr int STATUS_SMEM_ALIGN = 2;  // device status bit: shared memory base not alignable

struct BwdParams {
    const float *lse2;   // [B*H, n_pad] LSE * log2(e)
    const float *delta;  // [B*H, n_pad] dO . O
    int *status;
    int heads;           // H: query heads per batch
    int kv_heads;        // H_kv: key/value heads per batch (divides H)
    int n;
    int n_pad;           // n rounded up to a multiple of 128
    int num_k_tiles;     // ceil(n / 128)
    int num_q_tiles;     // ceil(n / 128)
    float scale;         // softmax scale (factor of dQ and dK)
    float scale_log2;    // scale * log2(e)
    int causal;
    int window;          // < 0: none
    int block;           // > 0: block-local mask (see Mask)
};

// Launch shape shared by both main kernels.
struct BwdRoles {
    static constexpr int THREADS = 384;
    static constexpr uint32_t REGS_LAUNCH = 168;
    static constexpr uint32_t REGS_SOFTMAX = 232;
    static constexpr uint32_t REGS_CTRL = 40;
    static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_CTRL == THREADS * REGS_LAUNCH,
                  "register split must use exactly the launch allocation");
};

// dK / dV kernel: K_j, V_j, a ring of NST (Q_i, dO_i, lse2_i, delta_i) stages.
template <int D>
struct BwdKVCfg : BwdRoles {
    static_assert(D == 64 || D == 128, "head size 64 or 128");
    static constexpr int TILE_BYTES = BM * D * 2;
    static constexpr int BOXES = D / BOX_COLS;
    static constexpr int NST = (D == 128) ? 2 : 4;
    static constexpr int K_OFF = 0;
    static constexpr int V_OFF = K_OFF + TILE_BYTES;
    static constexpr int Q_OFF = V_OFF + TILE_BYTES;         // + s * TILE_BYTES
    static constexpr int DO_OFF = Q_OFF + NST * TILE_BYTES;  // + s * TILE_BYTES
    static constexpr int STAT_OFF = DO_OFF + NST * TILE_BYTES;  // + s * 1024: lse2[128], delta[128]
    static constexpr int BAR_OFF = STAT_OFF + NST * 1024;
    // kv_full, q_full[NST], q_empty[NST], s_full, dp_full, p_ready, ds_ready, kv_done, drain
    static constexpr int NUM_BARS = 7 + 2 * NST;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + 1 KB alignment slack
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t S_COL = 0;     // S^T; P^T over [0,32) and [64,96)
    static constexpr uint32_t DP_COL = 128;  // dP^T; dS^T over [128,160) and [192,224)
    static constexpr uint32_t DV_COL = 256;
    static constexpr uint32_t DK_COL = 256 + D;
    static_assert(DK_COL + D <= TMEM_COLS, "TMEM budget");
};

// dQ kernel: Q_i and dO_i (copied into TMEM at the start), then K_j, V_j
// alternately in a ring of NSLOT tiles.
template <int D>
struct BwdQCfg : BwdRoles {
    static_assert(D == 64 || D == 128, "head size 64 or 128");
    static constexpr int TILE_BYTES = BM * D * 2;
    static constexpr int BOXES = D / BOX_COLS;
    static constexpr int NSLOT = (D == 128) ? 4 : 8;
    static constexpr int Q_OFF = 0;    // also the dQ staging buffer of the epilogue
    static constexpr int DO_OFF = TILE_BYTES;
    static constexpr int KV_OFF = 2 * TILE_BYTES;  // + slot * TILE_BYTES
    static constexpr int BAR_OFF = KV_OFF + NSLOT * TILE_BYTES;
    // qd_full, qd_tmem, kv_full[NSLOT], kv_empty[NSLOT], s_full, s_read, dp_full, ds_ready, dq_done, drain
    static constexpr int NUM_BARS = 8 + 2 * NSLOT;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t S_COL = 0;
    static constexpr uint32_t DP_COL = 128;  // dP; dS over [128,160) and [192,224)
    static constexpr uint32_t DQ_COL = 256;
    static constexpr uint32_t QA_COL = 256 + D;           // Q_i as MMA operand: D/2 columns
    static constexpr uint32_t DOA_COL = 256 + D + D / 2;  // dO_i likewise
    static_assert(DOA_COL + D / 2 <= TMEM_COLS, "TMEM budget");
};

// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completion counted on `bar` in bytes; issued by the lane whose `leader` is set.
__device__ __forceinline__ void bulk_load_if(uint32_t leader, uint32_t dst, const void *src,
                                             uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "setp.ne.b32 e, %4, 0;\n\t"
        "@e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar), "r"(leader)
        : "memory");
}

__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 ld_shared_u4(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// 2^x for the pair of P entries with index `pair` among a thread's 32 pairs
// (the polynomial for the first ATTN_BWD_EX2_EMU of every 16).
__device__ __forceinline__ void ex2_pair(int pair, float x0, float x1, float &e0, float &e1)
{
    if ((pair % 16) < ATTN_BWD_EX2_EMU) {
        ex2_poly_x2(x0, x1, e0, e1);
    } else {
        e0 = ex2_approx(x0);
        e1 = ex2_approx(x1);
    }
}

// ---------------------------------------------------------------------------
// 1. delta_i = dO_i . O_i (fp32 over the bf16 values) and lse2_i = LSE_i log2(e)
// for rows i < n of every head, 0 in the padding rows up to n_pad. D/8 lanes
// per row, 8 elements (16 bytes) per lane.
template <int D>
__global__ void __launch_bounds__(256)
    attn_bwd_prep_kernel(const __nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ dout,
                         const float *__restrict__ lse, float *__restrict__ lse2,
                         float *__restrict__ delta, int64_t bh_count, int n, int n_pad)
{
    constexpr int L = D / 8;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t row = t / L;        // padded row id bh * n_pad + i
    const int part = static_cast<int>(t % L);
    const bool valid = row < bh_count * n_pad;
    const int64_t bh = valid ? row / n_pad : 0;
    const int i = valid ? static_cast<int>(row % n_pad) : 0;
    const bool real = valid && i < n;
    float acc = 0.f;
    if (real) {
        const int64_t off = (bh * n + i) * D + part * 8;
        const uint4 ov = *reinterpret_cast<const uint4 *>(o + off);
        const uint4 dv = *reinterpret_cast<const uint4 *>(dout + off);
        const __nv_bfloat162 *o2 = reinterpret_cast<const __nv_bfloat162 *>(&ov);
        const __nv_bfloat162 *d2 = reinterpret_cast<const __nv_bfloat162 *>(&dv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 a = __bfloat1622float2(o2[e]);
            const float2 b = __bfloat1622float2(d2[e]);
            acc = fmaf(a.x, b.x, acc);
            acc = fmaf(a.y, b.y, acc);
        }
    }
#pragma unroll
    for (int w = L / 2; w >= 1; w /= 2) acc += __shfl_xor_sync(0xffffffffu, acc, w);
    if (valid && part == 0) {
        delta[row] = real ? acc : 0.f;
        lse2[row] = real ? lse[bh * n + i] * 1.4426950408889634f : 0.f;
    }
}

// Query tiles [qlo, qhi) holding a query that attends to some key of the key
// tile starting at k0 (k0 < n). Causal and window masks only (the kernels'
// specialisation without a block mask keeps this arithmetic).
__device__ __forceinline__ void query_tile_range(int k0, int n, int causal, int window, int &qlo,
                                                 int &qhi)
{
    const int nqt = (n + BM - 1) / BM;
    qlo = causal ? k0 / BM : (window >= 0 ? max(0, k0 - window) / BM : 0);
    qhi = nqt;
    if (window >= 0) {
        const int64_t last = min(static_cast<int64_t>(n) - 1, static_cast<int64_t>(k0) + BN - 1 + window);
        qhi = static_cast<int>(last / BM) + 1;
    }
}

// The same for any Mask (used with a block mask).
__device__ __forceinline__ void query_tile_range(int k0, const Mask &mk, int &qlo, int &qhi)
{
    qlo = mk.first_query(k0) / BM;
    qhi = mk.last_query(min(k0 + BN - 1, mk.n - 1)) / BM + 1;
}

// The key-tile kernels walk items it = 0, 1, ...: query tile qi = it % nq of
// the group's head g = it / nq. WALK_GROUPS false: one head, qi = it (the
// counters stay out of the instantiation for multi-head attention).
template <bool WALK_GROUPS>
__device__ __forceinline__ void next_item(int &qi, int &g, int nq)
{
    if constexpr (WALK_GROUPS) {
        if (++qi == nq) {
            qi = 0;
            ++g;
        }
    } else {
        ++qi;
    }
}



// Dynamic shared memory base rounded up to 1 KB (the 128-byte swizzle atoms
// need it); false if the slack does not allow it (never with the 1 KB of
// slack both kernels request; the caller then returns before touching any
// barrier or TMEM).
__device__ __forceinline__ bool smem_base_1k(uint8_t *raw_ptr, uint32_t &base, uint8_t *&base_ptr)
{
    const uint32_t raw = smem_addr(raw_ptr);
    base = (raw + 1023u) & ~1023u;
    base_ptr = raw_ptr + (base - raw);
    return base - raw <= 1024u;
}

// ---------------------------------------------------------------------------
// 2. dK and dV. GENERAL: compiled for grouped-query heads (kv_heads <
// heads) or the block-local mask (block > 0); the other instantiation handles
// multi-head attention under the causal and window masks. NOMASK (never with
// GENERAL): compiled without the mask test, for problems with no mask whose
// length is a whole number of tiles (no tile needs one; the test, never
// taken there, still cost 2%).
template <int D, bool GENERAL, bool NOMASK>
__global__ void __launch_bounds__(BwdRoles::THREADS, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                         const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                         const BwdParams p)
{
    using C = BwdKVCfg<D>;
    constexpr int NST = C::NST;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint32_t base;
    uint8_t *base_ptr;
    if (!smem_base_1k(smem_raw, base, base_ptr)) {
        if (threadIdx.x == 0) atomicOr(p.status, STATUS_SMEM_ALIGN);
        return;
    }
    const uint32_t sK = base + C::K_OFF, sV = base + C::V_OFF;
    auto sQ = [&](int s) { return base + C::Q_OFF + s * C::TILE_BYTES; };
    auto sdO = [&](int s) { return base + C::DO_OFF + s * C::TILE_BYTES; };
    auto sStat = [&](int s) { return base + C::STAT_OFF + s * 1024; };
    const uint32_t bars = base + C::BAR_OFF;
    const uint32_t kv_full = bars;
    auto q_full = [&](int s) { return bars + 8u * (1 + s); };
    auto q_empty = [&](int s) { return bars + 8u * (1 + NST + s); };
    const uint32_t s_full = bars + 8u * (1 + 2 * NST);
    const uint32_t dp_full = s_full + 8, p_ready = s_full + 16, ds_ready = s_full + 24;
    const uint32_t kv_done = s_full + 32, drain_bar = s_full + 40;
    uint32_t *const tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + C::MISC_OFF);
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(base_ptr + C::MISC_OFF + 4);

    const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x / 32), 0);

    // Work: the key tiles of one key/value head are adjacent in blockIdx (Q /
    // dO reuse in L2); under a causal mask the early key tiles (most query
    // tiles) first. The CTA walks the query tiles [qlo, qhi) of every query
    // head of the group (grouped-query attention: G = H / H_kv heads share
    // this key/value head; G = 1 for multi-head attention), item it being
    // query tile qlo + it % nq of the group's head it / nq.
    const int bkv = blockIdx.x / p.num_k_tiles;
    const int kt = static_cast<int>(blockIdx.x % p.num_k_tiles);
    const int k0 = kt * BN;
    const int n = p.n;
    const int G = p.heads / p.kv_heads;
    const int bh0 = (bkv / p.kv_heads) * p.heads + (bkv % p.kv_heads) * G;  // first query head
    int qlo, qhi;
    if constexpr (GENERAL)
        query_tile_range(k0, Mask{n, p.causal, p.window, p.block}, qlo, qhi);
    else
        query_tile_range(k0, n, p.causal, p.window, qlo, qhi);
    const int nq = qhi - qlo;  // >= 1: query k0 attends to key k0
    const int nitems = GENERAL ? G * nq : nq;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < NST; ++s) {
            mbar_init(q_full(s), 1);
            mbar_init(q_empty(s), 1);
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(p_ready, 2 * BN);
        mbar_init(ds_ready, 2 * BN);
        mbar_init(kv_done, 1);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9 && (threadIdx.x % 32) == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
    }
    if (warp == 8) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Waiter wt{abort_flag, p.status};

    if (warp >= 8) {
      regs_decrease<C::REGS_CTRL>();
      const uint32_t leader = elect_one();
      if (warp == 9) {
        // ------------------------------------------------------------ TMA producer
        mbar_arrive_expect_tx_if(leader, kv_full, 2 * C::TILE_BYTES);
#pragma unroll
        for (int b = 0; b < C::BOXES; ++b) {
            tma_load_3d_if(leader, sK + b * BOX_BYTES, &tmK, kv_full, b * BOX_COLS, k0, bkv);
            tma_load_3d_if(leader, sV + b * BOX_BYTES, &tmV, kv_full, b * BOX_COLS, k0, bkv);
        }
        int issued = 0;
        // (qi, g) = (it % nq, it / nq), kept by increment
        for (int it = 0, qi = 0, g = 0; it < nitems; ++it, next_item<GENERAL>(qi, g, nq)) {
            const int s = it % NST;
            if (it >= NST && !__all_sync(0xffffffffu, wt.wait(q_empty(s), ((it / NST) & 1u) ^ 1u)))
                break;
            const int q0 = (qlo + qi) * BM;
            const int bh = bh0 + g;
#ifdef ATTN_FAULT_BWD_DROP_FIRST_Q
            // Test hook (never defined in the library build): the first Q/dO
            // stage is never loaded, so the MMA warp's wait on it must expire
            // and the kernel must stop cleanly.
            if (it == 0) {
                ++issued;
                continue;
            }
#endif
            mbar_arrive_expect_tx_if(leader, q_full(s), 2 * C::TILE_BYTES + 1024);
#pragma unroll
            for (int b = 0; b < C::BOXES; ++b) {
                tma_load_3d_if(leader, sQ(s) + b * BOX_BYTES, &tmQ, q_full(s), b * BOX_COLS, q0, bh);
                tma_load_3d_if(leader, sdO(s) + b * BOX_BYTES, &tmdO, q_full(s), b * BOX_COLS, q0, bh);
            }
            const size_t srow = static_cast<size_t>(bh) * p.n_pad + q0;
            bulk_load_if(leader, sStat(s), p.lse2 + srow, 512, q_full(s));
            bulk_load_if(leader, sStat(s) + 512, p.delta + srow, 512, q_full(s));
            ++issued;
        }
        // Let every copy issued into shared memory land before teardown (the
        // MMA warp may have stopped early): the last load of each stage.
        wt.drain(kv_full, 0);
        for (int s = 0; s < NST; ++s)
            if (issued > s) wt.drain(q_full(s), ((issued - 1 - s) / NST) & 1u);
      } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc_t = idesc_bf16_f32(BN, BM, 0, 0);  // S^T, dP^T: both K-major
        constexpr uint32_t idesc_acc = idesc_bf16_f32(BN, D, 0, 1); // dV, dK: A in TMEM, B MN-major
        bool ok = __all_sync(0xffffffffu, wt.wait(kv_full, 0));
        tc_fence_after();
        const uint64_t k_kmaj = smem_desc_sw128(sK, 16, 1024);
        const uint64_t v_kmaj = smem_desc_sw128(sV, 16, 1024);
        auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
            if (!__all_sync(0xffffffffu, wt.wait(bar, parity))) return false;
            tc_fence_after();
            return true;
        };
        // S^T(it) = K Q_it^T: D/16 MMAs over the head dimension
        auto issue_s = [&](int it) {
            const uint64_t q_kmaj = smem_desc_sw128(sQ(it % NST), 16, 1024);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint64_t off = static_cast<uint64_t>(((k / 4) * BOX_BYTES + (k % 4) * 32) >> 4);
                mma_bf16_ss_if(leader, tmem + C::S_COL, k_kmaj + off, q_kmaj + off, idesc_t, k > 0 ? 1u : 0u);
            }
            mma_commit_if(leader, s_full);
        };
        // dP^T(it) = V dO_it^T
        auto issue_dp = [&](int it) {
            const uint64_t do_kmaj = smem_desc_sw128(sdO(it % NST), 16, 1024);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint64_t off = static_cast<uint64_t>(((k / 4) * BOX_BYTES + (k % 4) * 32) >> 4);
                mma_bf16_ss_if(leader, tmem + C::DP_COL, v_kmaj + off, do_kmaj + off, idesc_t, k > 0 ? 1u : 0u);
            }
            mma_commit_if(leader, dp_full);
        };
        // Issue order: S(0), dP(0), then per query tile it
        //   dV(it), S(it+1), dK(it), dP(it+1).
        // S(it+1) overwrites P^T(it) right behind dV(it), its reader, and
        // dP(it+1) overwrites dS^T(it) right behind dK(it) (MMAs complete in
        // issue order), so the softmax warps can start on tile it+1 as soon
        // as they have produced dS^T(it).
        if (ok) ok = wait(q_full(0), 0);
        if (ok) {
            issue_s(0);
            issue_dp(0);
        }
        for (int it = 0; ok && it < nitems; ++it) {
            const int s = it % NST;
            const uint64_t q_mn = smem_desc_sw128(sQ(s), BOX_BYTES, 1024);
            const uint64_t do_mn = smem_desc_sw128(sdO(s), BOX_BYTES, 1024);
            // dV += P^T dO: 8 MMAs of 16 queries; P^T of queries [0,64) is in
            // TMEM columns [0,32), of queries [64,128) in [64,96)
            if (!(ok = wait(p_ready, it & 1u))) break;
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk) {
                const uint32_t pcol = (kk < 4) ? kk * 8 : 64 + (kk - 4) * 8;
                mma_bf16_ts_if(leader, tmem + C::DV_COL, tmem + C::S_COL + pcol,
                               do_mn + static_cast<uint64_t>(kk * 128), idesc_acc,
                               (it > 0 || kk > 0) ? 1u : 0u);
            }
            if (it + 1 < nitems) {
                if (!(ok = wait(q_full((it + 1) % NST), ((it + 1) / NST) & 1u))) break;
                issue_s(it + 1);
            }
            // dK += dS^T Q: dS^T in TMEM like P^T, in dP^T's columns
            if (!(ok = wait(ds_ready, it & 1u))) break;
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk) {
                const uint32_t dcol = (kk < 4) ? kk * 8 : 64 + (kk - 4) * 8;
                mma_bf16_ts_if(leader, tmem + C::DK_COL, tmem + C::DP_COL + dcol,
                               q_mn + static_cast<uint64_t>(kk * 128), idesc_acc,
                               (it > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit_if(leader, q_empty(s));
            if (it + 1 < nitems) issue_dp(it + 1);
        }
        if (ok) mma_commit_if(leader, kv_done);
        // Every MMA this warp issued must finish before TMEM is freed.
        mma_commit_if(leader, drain_bar);
        wt.drain(drain_bar, 0);
      }
    } else {
        // ------------------------------------------------------------ softmax / dS
        regs_increase<C::REGS_SOFTMAX>();
        const int h = warp / 4;                 // query columns [64h, 64h + 64)
        const int r = threadIdx.x % BN;         // key row in the tile == TMEM lane
        const int key = k0 + r;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
        const float sc = p.scale_log2;
        const int causal = p.causal, window = p.window;
        // Block mask: bounds that do not change along the query walk (this
        // key's attending queries, and the bounds every key of the tile
        // shares).
        const Mask mk{n, p.causal, p.window, p.block};
        const int key_first = mk.first_query(key), key_last = (key < n) ? mk.last_query(key) : -1;
        const int tile_first = mk.first_query(min(k0 + BN - 1, n - 1)), tile_last = mk.last_query(k0);
        const bool tile_ragged = k0 + BN > n;
        bool ok = true;
        for (int it = 0, qi = 0, g = 0; it < nitems; ++it, next_item<GENERAL>(qi, g, nq)) {
            const int s = it % NST;
            const int q0 = (qlo + qi) * BM;
            ok = __all_sync(0xffffffffu, wt.wait(s_full, it & 1u));
            if (!ok) break;
            tc_fence_after();
            // Allowed query columns of this key row: one interval [lo, hi].
            bool need_mask;
            int lo, hi;
            if constexpr (GENERAL) {
                need_mask = tile_ragged || (q0 + BM > n) || tile_first > q0 || tile_last < q0 + BM - 1;
                lo = key_first - q0;
                hi = (key < n) ? key_last - q0 : -1;
            } else {
                need_mask = !NOMASK && ((k0 + BN > n) || (q0 + BM > n) || (causal && q0 < k0 + BN - 1) ||
                                        (window >= 0 && q0 + BM - 1 > k0 + window) ||
                                        (!causal && window >= 0 && q0 < k0 + BN - 1 - window));
                lo = causal ? key - q0 : (window >= 0 ? key - window - q0 : 0);
                hi = min(BM - 1, n - 1 - q0);
                if (window >= 0) hi = min(hi, key + window - q0);
                if (key >= n) hi = -1;
            }
            const uint32_t stat = sStat(s);
            float pf[64];
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                const int cb = 64 * h + 32 * c2;  // first query column of this chunk
                uint32_t sv[32];
                tmem_ld32(lane_base + C::S_COL + cb, sv);
                uint32_t pk[16];
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const float4 l4 = ld_shared_f4(stat + (cb + 4 * g) * 4);
                    const float2 x01 = ffma2(make_float2(u2f(sv[4 * g]), u2f(sv[4 * g + 1])),
                                             make_float2(sc, sc), make_float2(-l4.x, -l4.y));
                    const float2 x23 = ffma2(make_float2(u2f(sv[4 * g + 2]), u2f(sv[4 * g + 3])),
                                             make_float2(sc, sc), make_float2(-l4.z, -l4.w));
                    float e[4];
                    ex2_pair(16 * c2 + 2 * g, x01.x, x01.y, e[0], e[1]);
                    ex2_pair(16 * c2 + 2 * g + 1, x23.x, x23.y, e[2], e[3]);
                    if (need_mask) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int c = cb + 4 * g + u;
                            if (c < lo || c > hi) e[u] = 0.f;
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) pf[32 * c2 + 4 * g + u] = e[u];
                    pk[2 * g] = pack_bf16x2(e[0], e[1]);
                    pk[2 * g + 1] = pack_bf16x2(e[2], e[3]);
                }
                // P^T over this thread's own, already read, S^T columns
                tmem_st16(lane_base + C::S_COL + 64 * h + 16 * c2, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_ready);

            ok = __all_sync(0xffffffffu, wt.wait(dp_full, it & 1u));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                const int cb = 64 * h + 32 * c2;
                uint32_t dv[32];
                tmem_ld32(lane_base + C::DP_COL + cb, dv);
                uint32_t pk[16];
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const float4 d4 = ld_shared_f4(stat + 512 + (cb + 4 * g) * 4);
                    const float2 t01 = fsub2(make_float2(u2f(dv[4 * g]), u2f(dv[4 * g + 1])), make_float2(d4.x, d4.y));
                    const float2 t23 = fsub2(make_float2(u2f(dv[4 * g + 2]), u2f(dv[4 * g + 3])), make_float2(d4.z, d4.w));
                    const float2 s01 = fmul2(t01, make_float2(pf[32 * c2 + 4 * g], pf[32 * c2 + 4 * g + 1]));
                    const float2 s23 = fmul2(t23, make_float2(pf[32 * c2 + 4 * g + 2], pf[32 * c2 + 4 * g + 3]));
                    pk[2 * g] = pack_bf16x2(s01.x, s01.y);
                    pk[2 * g + 1] = pack_bf16x2(s23.x, s23.y);
                }
                // dS^T over this thread's own, already read, dP^T columns
                tmem_st16(lane_base + C::DP_COL + 64 * h + 16 * c2, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ds_ready);
        }
        if (ok) ok = __all_sync(0xffffffffu, wt.wait(kv_done, 0));
        const bool all_ok = named_bar_and(1 + h, BN, ok);
        if (all_ok) {
            tc_fence_after();
            // dV (h = 0) or scale * dK (h = 1): TMEM -> bf16 -> swizzled smem
            // (a Q / dO ring stage, idle once every MMA is done) -> TMA store;
            // rows past n are clipped by the store.
            const uint32_t col = h ? C::DK_COL : C::DV_COL;
            const float mul = h ? p.scale : 1.f;
            const uint32_t stage = h ? sdO(0) : sQ(0);
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
                uint32_t v[32];
                tmem_ld32(lane_base + col + c, v);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(u2f(v[2 * i]) * mul, u2f(v[2 * i + 1]) * mul);
                const uint32_t rowp = stage + (c / BOX_COLS) * BOX_BYTES + r * 128;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint32_t chunk = static_cast<uint32_t>((c % BOX_COLS) / 8 + q4) ^ static_cast<uint32_t>(r & 7);
                    st_shared_v4(rowp + chunk * 16, pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(1 + h, BN);
            if (r == 0) {
                const CUtensorMap *map = h ? &tmdK : &tmdV;
                for (int b = 0; b < C::BOXES; ++b) tma_store_3d(map, stage + b * BOX_BYTES, b * BOX_COLS, k0, bkv);
                tma_store_commit();
                tma_store_wait_read0();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// 3. dQ.
// GENERAL and NOMASK as for attn_bwd_dkdv_kernel (here only the mask
// arithmetic differs: the head mapping is the same for both).
template <int D, bool GENERAL, bool NOMASK>
__global__ void __launch_bounds__(BwdRoles::THREADS, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmdQ, const BwdParams p)
{
    using C = BwdQCfg<D>;
    constexpr int NSLOT = C::NSLOT;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint32_t base;
    uint8_t *base_ptr;
    if (!smem_base_1k(smem_raw, base, base_ptr)) {
        if (threadIdx.x == 0) atomicOr(p.status, STATUS_SMEM_ALIGN);
        return;
    }
    const uint32_t sQ = base + C::Q_OFF, sdO = base + C::DO_OFF;
    auto sKV = [&](int slot) { return base + C::KV_OFF + slot * C::TILE_BYTES; };
    const uint32_t bars = base + C::BAR_OFF;
    const uint32_t qd_full = bars, qd_tmem = bars + 8;
    auto kv_full = [&](int slot) { return bars + 8u * (2 + slot); };
    auto kv_empty = [&](int slot) { return bars + 8u * (2 + NSLOT + slot); };
    const uint32_t s_full = bars + 8u * (2 + 2 * NSLOT);
    const uint32_t s_read = s_full + 8, dp_full = s_full + 16, ds_ready = s_full + 24;
    const uint32_t dq_done = s_full + 32, drain_bar = s_full + 40;
    uint32_t *const tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + C::MISC_OFF);
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(base_ptr + C::MISC_OFF + 4);

    const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x / 32), 0);

    // Work: query tiles of one head adjacent in blockIdx (K / V reuse in L2);
    // within a head the late tiles (the most key tiles under a causal mask)
    // first.
    const int bh = blockIdx.x / p.num_q_tiles;
    // key/value head of this query head (grouped-query attention)
    const int bkv = (bh / p.heads) * p.kv_heads + (bh % p.heads) / (p.heads / p.kv_heads);
    const int qt = p.num_q_tiles - 1 - static_cast<int>(blockIdx.x % p.num_q_tiles);
    const int q0 = qt * BM;
    const int n = p.n;
    int jlo, jhi;
    if constexpr (GENERAL)
        key_tile_range(q0, Mask{n, p.causal, p.window, p.block}, jlo, jhi);
    else
        key_tile_range(q0, n, p.causal, p.window, jlo, jhi);
    const int nkv = jhi - jlo;  // >= 1: key q0 is allowed for query q0

    if (threadIdx.x == 0) {
        mbar_init(qd_full, 1);
        mbar_init(qd_tmem, 2 * BM);
        for (int i = 0; i < NSLOT; ++i) {
            mbar_init(kv_full(i), 1);
            mbar_init(kv_empty(i), 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_read, 2 * BM);
        mbar_init(dp_full, 1);
        mbar_init(ds_ready, 2 * BM);
        mbar_init(dq_done, 1);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9 && (threadIdx.x % 32) == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
        tma_prefetch_desc(&tmdQ);
    }
    if (warp == 8) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Waiter wt{abort_flag, p.status};

    if (warp >= 8) {
      regs_decrease<C::REGS_CTRL>();
      const uint32_t leader = elect_one();
      if (warp == 9) {
        // ------------------------------------------------------------ TMA producer
        mbar_arrive_expect_tx_if(leader, qd_full, 2 * C::TILE_BYTES);
#pragma unroll
        for (int b = 0; b < C::BOXES; ++b) {
            tma_load_3d_if(leader, sQ + b * BOX_BYTES, &tmQ, qd_full, b * BOX_COLS, q0, bh);
            tma_load_3d_if(leader, sdO + b * BOX_BYTES, &tmdO, qd_full, b * BOX_COLS, q0, bh);
        }
        // item i: K of key tile jlo + i/2 (i even) or V of it (i odd)
        int issued = 0;
        for (int i = 0; i < 2 * nkv; ++i) {
            const int slot = i % NSLOT;
            if (i >= NSLOT &&
                !__all_sync(0xffffffffu, wt.wait(kv_empty(slot), ((i / NSLOT) & 1u) ^ 1u)))
                break;
            mbar_arrive_expect_tx_if(leader, kv_full(slot), C::TILE_BYTES);
            const CUtensorMap *map = (i & 1) ? &tmV : &tmK;
            const int k0 = (jlo + i / 2) * BN;
#pragma unroll
            for (int b = 0; b < C::BOXES; ++b)
                tma_load_3d_if(leader, sKV(slot) + b * BOX_BYTES, map, kv_full(slot), b * BOX_COLS, k0, bkv);
            ++issued;
        }
        wt.drain(qd_full, 0);
        for (int slot = 0; slot < NSLOT; ++slot)
            if (issued > slot) wt.drain(kv_full(slot), ((issued - 1 - slot) / NSLOT) & 1u);
      } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc_s = idesc_bf16_f32(BM, BN, 0, 0);  // S, dP: A in TMEM, B K-major
        constexpr uint32_t idesc_dq = idesc_bf16_f32(BM, D, 0, 1);  // dQ: A in TMEM, B MN-major
        auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
            if (!__all_sync(0xffffffffu, wt.wait(bar, parity))) return false;
            tc_fence_after();
            return true;
        };
        // ring item of K_t (2t) or V_t (2t + 1): its slot and the parity of its load
        auto slot_of = [&](int item) { return item % NSLOT; };
        auto par_of = [&](int item) { return static_cast<uint32_t>((item / NSLOT) & 1); };
        // S(t) = Q K_t^T: A = Q from TMEM (D/2 columns, 8 per 16-wide K step)
        auto issue_s = [&](int t) -> bool {
            const int ik = 2 * t;
            if (!wait(kv_full(slot_of(ik)), par_of(ik))) return false;
            const uint64_t kdesc = smem_desc_sw128(sKV(slot_of(ik)), 16, 1024);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint64_t off = static_cast<uint64_t>(((k / 4) * BOX_BYTES + (k % 4) * 32) >> 4);
                mma_bf16_ts_if(leader, tmem + C::S_COL, tmem + C::QA_COL + k * 8, kdesc + off, idesc_s,
                               k > 0 ? 1u : 0u);
            }
            mma_commit_if(leader, s_full);
            return true;
        };
        // dP(t) = dO V_t^T
        auto issue_dp = [&](int t) -> bool {
            const int iv = 2 * t + 1;
            if (!wait(kv_full(slot_of(iv)), par_of(iv))) return false;
            const uint64_t vdesc = smem_desc_sw128(sKV(slot_of(iv)), 16, 1024);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint64_t off = static_cast<uint64_t>(((k / 4) * BOX_BYTES + (k % 4) * 32) >> 4);
                mma_bf16_ts_if(leader, tmem + C::DP_COL, tmem + C::DOA_COL + k * 8, vdesc + off, idesc_s,
                               k > 0 ? 1u : 0u);
            }
            mma_commit_if(leader, dp_full);
            return true;
        };
        // Issue order: S(0), dP(0), then per key tile t
        //   S(t+1) once the softmax has read S(t); dQ(t), dP(t+1) once dS(t) is in TMEM.
        // dS(t) sits in dP's columns; dP(t+1) overwrites it right behind
        // dQ(t), its reader (MMAs complete in issue order).
        bool ok = wait(qd_tmem, 0);
        if (ok) ok = issue_s(0);
        if (ok) ok = issue_dp(0);
        for (int t = 0; ok && t < nkv; ++t) {
            if (t + 1 < nkv) {
                if (!(ok = wait(s_read, t & 1u))) break;
                if (!(ok = issue_s(t + 1))) break;
            }
            if (!(ok = wait(ds_ready, t & 1u))) break;
            // dQ += dS K_t: dS of keys [0,64) in TMEM columns [128,160), of
            // keys [64,128) in [192,224); K_t read MN-major (keys along K)
            const int ik = 2 * t;
            const uint64_t kmn = smem_desc_sw128(sKV(slot_of(ik)), BOX_BYTES, 1024);
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
                const uint32_t dcol = (kk < 4) ? kk * 8 : 64 + (kk - 4) * 8;
                mma_bf16_ts_if(leader, tmem + C::DQ_COL, tmem + C::DP_COL + dcol,
                               kmn + static_cast<uint64_t>(kk * 128), idesc_dq, (t > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit_if(leader, kv_empty(slot_of(ik)));
            mma_commit_if(leader, kv_empty(slot_of(ik + 1)));
            if (t + 1 < nkv && !(ok = issue_dp(t + 1))) break;
        }
        if (ok) mma_commit_if(leader, dq_done);
        mma_commit_if(leader, drain_bar);
        wt.drain(drain_bar, 0);
      }
    } else {
        // ------------------------------------------------------------ softmax / dS
        regs_increase<C::REGS_SOFTMAX>();
        const int h = warp / 4;                 // key columns [64h, 64h + 64)
        const int r = threadIdx.x % BM;         // query row in the tile == TMEM lane
        const int row = q0 + r;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
        const float sc = p.scale_log2;
        const int causal = p.causal, window = p.window;
        // Block mask: bounds that do not change along the key walk.
        const Mask mk{n, p.causal, p.window, p.block};
        const int row_first = mk.first_key(row), row_last = mk.last_key(row);
        const int tile_first = mk.first_key(q0 + BM - 1), tile_last = mk.last_key(q0);
        // this row's log2-domain LSE and delta (0 in rows past n)
        const size_t srow = static_cast<size_t>(bh) * p.n_pad + row;
        const float nl2 = -p.lse2[srow];
        const float dlt = p.delta[srow];
        // Q (h = 0) or dO (h = 1) row r -> TMEM as the A operand of S or dP:
        // lane r, two bf16 per column, read out of the 128-byte swizzled tile.
        bool ok = __all_sync(0xffffffffu, wt.wait(qd_full, 0));
        if (ok) {
            const uint32_t src = h ? sdO : sQ;
            const uint32_t dst = lane_base + (h ? C::DOA_COL : C::QA_COL);
#pragma unroll
            for (int b = 0; b < C::BOXES; ++b) {
                uint32_t v[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t chunk = static_cast<uint32_t>(j) ^ static_cast<uint32_t>(r & 7);
                    const uint4 u = ld_shared_u4(src + b * BOX_BYTES + r * 128 + chunk * 16);
                    v[4 * j] = u.x;
                    v[4 * j + 1] = u.y;
                    v[4 * j + 2] = u.z;
                    v[4 * j + 3] = u.w;
                }
                tmem_st32(dst + b * 32, v);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(qd_tmem);
        }
        for (int t = 0; ok && t < nkv; ++t) {
            const int k0 = (jlo + t) * BN;
            ok = __all_sync(0xffffffffu, wt.wait(s_full, t & 1u));
            if (!ok) break;
            tc_fence_after();
            uint32_t sa[32], sb[32];
            tmem_ld32(lane_base + C::S_COL + 64 * h, sa);
            tmem_ld32(lane_base + C::S_COL + 64 * h + 32, sb);
            // S(t) is in registers: the MMA warp may compute S(t+1)
            tc_fence_before();
            mbar_arrive(s_read);
            const bool need_mask =
                !NOMASK && (GENERAL ? ((k0 + BN > n) || tile_first > k0 || tile_last < k0 + BN - 1)
                                    : ((k0 + BN > n) || (causal && k0 + BN - 1 > q0) ||
                                       (window >= 0 && k0 < q0 + BM - 1 - window) ||
                                       (!causal && window >= 0 && k0 + BN - 1 > q0 + window)));
            // allowed key columns of this row: [lo, hi], key = k0 + column
            const int hi = GENERAL ? row_last - k0
                                     : min(causal ? row - k0 : (window >= 0 ? row + window - k0 : BN - 1),
                                           n - 1 - k0);
            const int lo = GENERAL ? row_first - k0 : ((window >= 0) ? row - window - k0 : 0);
            float pf[64];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const uint32_t s0 = (i < 16) ? sa[2 * i] : sb[2 * i - 32];
                const uint32_t s1 = (i < 16) ? sa[2 * i + 1] : sb[2 * i - 31];
                const float2 x = ffma2(make_float2(u2f(s0), u2f(s1)), make_float2(sc, sc), make_float2(nl2, nl2));
                ex2_pair(i, x.x, x.y, pf[2 * i], pf[2 * i + 1]);
            }
            if (need_mask) {
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    const int c = 64 * h + i;
                    if (c < lo || c > hi) pf[i] = 0.f;
                }
            }
            ok = __all_sync(0xffffffffu, wt.wait(dp_full, t & 1u));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                uint32_t dv[32];
                tmem_ld32(lane_base + C::DP_COL + 64 * h + 32 * c2, dv);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 tt = fsub2(make_float2(u2f(dv[2 * i]), u2f(dv[2 * i + 1])), make_float2(dlt, dlt));
                    const float2 ds = fmul2(tt, make_float2(pf[32 * c2 + 2 * i], pf[32 * c2 + 2 * i + 1]));
                    pk[i] = pack_bf16x2(ds.x, ds.y);
                }
                // dS over this thread's own, already read, dP columns
                tmem_st16(lane_base + C::DP_COL + 64 * h + 16 * c2, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ds_ready);
        }
        if (ok) ok = __all_sync(0xffffffffu, wt.wait(dq_done, 0));
        const bool all_ok = named_bar_and(1, 2 * BM, ok);
        if (all_ok) {
            tc_fence_after();
            // scale * dQ: warpgroup h stores columns [h*D/2, (h+1)*D/2) of row
            // r -> bf16 -> swizzled smem (the Q tile, unused since it was
            // copied into TMEM) -> TMA store; rows past n are clipped.
            const float mul = p.scale;
#pragma unroll 1
            for (int c = h * (D / 2); c < (h + 1) * (D / 2); c += 32) {
                uint32_t v[32];
                tmem_ld32(lane_base + C::DQ_COL + c, v);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(u2f(v[2 * i]) * mul, u2f(v[2 * i + 1]) * mul);
                const uint32_t rowp = sQ + (c / BOX_COLS) * BOX_BYTES + r * 128;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint32_t chunk = static_cast<uint32_t>((c % BOX_COLS) / 8 + q4) ^ static_cast<uint32_t>(r & 7);
                    st_shared_v4(rowp + chunk * 16, pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 2 * BM);
            if (threadIdx.x == 0) {
                for (int b = 0; b < C::BOXES; ++b) tma_store_3d(&tmdQ, sQ + b * BOX_BYTES, b * BOX_COLS, q0, bh);
                tma_store_commit();
                tma_store_wait_read0();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace attn_sm100
