// attn_bwd_fused_kernel.cuh - the backward pass as one key-tile kernel, with
// dQ added into an fp32 accumulator by TMA reduce-adds. Used for head size
// 64: there the split kernels of attn_bwd_kernel.cuh (dQ in a kernel of its
// own, which recomputes the exponentials) are bound by the exponential unit
// and measured slower than this kernel, which is bound by the L2's reduction
// throughput instead.
//
// The gradients, the recompute and the roles are those described in
// attn_bwd_kernel.cuh; this file differs in:
//   2. attn_bwd_fused_kernel: one CTA per (batch * key/value head, 128-key
//      tile), walking the query tiles of every query head of the group. Per
//      query tile it runs five tcgen05 MMAs:
//        S^T  = K_j Q_i^T        (smem x smem -> TMEM, 128 keys x 128 queries)
//        dP^T = V_j dO_i^T       (smem x smem -> TMEM)
//        dV  += P^T dO_i         (P^T from TMEM, written there by the softmax warps)
//        dK  += dS^T Q_i         (dS^T from shared memory, K-major)
//        dQ_i = dS K_j           (the same dS buffer read MN-major)
//      and adds each dQ_i tile into the fp32 accumulator.
//   1./3. attn_bwd_fused_prep_kernel also zeroes the accumulator, and
//      attn_bwd_dq_convert_kernel turns it into bf16 dQ.
//
// Roles (512 threads, 16 warps = 4 warpgroups):
//   warps 0-3, 4-7  "softmax": thread r of warpgroup h owns key row r (TMEM
//                   lane r) and query columns [64h, 64h+64) of the tile. It
//                   turns S^T into P^T (written back into TMEM over its own S
//                   columns) and dP^T into dS^T (bf16, into the swizzled dS
//                   buffer); after the walk it stores dV (h = 0) or dK (h = 1).
//   warp 8          MMA issuer (one elected lane) and TMEM owner.
//   warp 9          TMA producer: K_j, V_j once, then Q_i, dO_i and the rows'
//                   LSE and delta into a two-stage ring.
//   warps 10-11     idle.
//   warps 12-15     dQ drain: TMEM -> registers (times scale) -> swizzled fp32
//                   staging in shared memory -> TMA reduce-add into the
//                   accumulator, 64 columns (32 KB) at a time.
// Registers: launched at 128 per thread; the softmax warpgroups raise to 184,
// the dQ warpgroup drops to 88 and the MMA/TMA warpgroup to 56
// (2*184 + 88 + 56 = 4*128).
#pragma once
#include "attn_bwd_kernel.cuh"

namespace attn_sm100 {

constexpr int FUSED_BWD_NSTAGE = 2;              // Q_i / dO_i ring stages

struct FusedBwdParams {
    float *dq_acc;       // [B*H, n, d] fp32, zeroed by the prep kernel
    const float *lse2;   // [B*H, n_pad] LSE * log2(e)
    const float *delta;  // [B*H, n_pad] dO . O
    int *status;
    int heads;           // H: query heads per batch
    int kv_heads;        // H_kv: key/value heads per batch (divides H)
    int n;
    int n_pad;           // n rounded up to a multiple of 128
    int num_k_tiles;     // ceil(n / 128)
    float scale;         // softmax scale (factor of dQ and dK)
    float scale_log2;    // scale * log2(e)
    int causal;
    int window;          // < 0: none
    int block;           // > 0: block-local mask (see Mask)
};

template <int D>
struct FusedBwdCfg {
    static_assert(D == 64 || D == 128, "head size 64 or 128");
    static constexpr int TILE_BYTES = BM * D * 2;
    static constexpr int BOXES = D / BOX_COLS;
    static constexpr int NST = FUSED_BWD_NSTAGE;
    static constexpr int DS_BYTES = BN * BM * 2;  // 128 keys x 128 queries bf16
    static constexpr int K_OFF = 0;
    static constexpr int V_OFF = K_OFF + TILE_BYTES;
    static constexpr int Q_OFF = V_OFF + TILE_BYTES;        // + s * TILE_BYTES
    static constexpr int DO_OFF = Q_OFF + NST * TILE_BYTES;  // + s * TILE_BYTES
    static constexpr int DS_OFF = DO_OFF + NST * TILE_BYTES;
    static constexpr int STAT_OFF = DS_OFF + DS_BYTES;       // + s * 1024: lse2[128], delta[128]
    // dQ staging for the TMA reduce-add: 64 fp32 columns of the 128 query
    // rows (32 KB, two 128-byte swizzled boxes of 32 columns). D = 64 has a
    // buffer of its own; D = 128 has no room left and stages its two halves
    // in the dS buffer, which is idle from the end of dQ_i's MMA until the
    // softmax writes dS_{i+1}.
    static constexpr bool DQ_IN_DS = (D == 128);
    static constexpr int DQS_HALF_BYTES = BM * 64 * 4;
    static constexpr int DQS_OWN_OFF = STAT_OFF + NST * 1024;
    static constexpr int BAR_OFF = DQS_OWN_OFF + (DQ_IN_DS ? 0 : DQS_HALF_BYTES);
    static constexpr int DQS_OFF = DQ_IN_DS ? DS_OFF : DQS_OWN_OFF;
    // kv_full, q_full[NST], q_empty[NST], s_full, dp_full, p_ready, ds_ready,
    // dq_full, dq_free, ds_free, kv_done, drain, dqs_free
    static constexpr int NUM_BARS = 11 + 2 * NST;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int SMEM_USED = MISC_OFF + 16;
    // Slack for aligning the dynamic shared memory base to 1024 bytes (the
    // 128-byte swizzle atoms need it); at D = 128 less than 1 KB is left.
    static constexpr int SLACK = (232448 - SMEM_USED >= 1024) ? 1024 : ((232448 - SMEM_USED) & ~127);
    static constexpr int SMEM_BYTES = SMEM_USED + SLACK;
    static_assert(SLACK >= 128 && SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t S_COL = 0;     // S^T, then P^T in [0,32) and [64,96)
    static constexpr uint32_t DP_COL = 128;  // dP^T
    static constexpr uint32_t DV_COL = 256;
    static constexpr uint32_t DK_COL = 256 + D;
    // dQ_i: D = 64 has columns of its own; D = 128 reuses dP^T's once the
    // softmax warps have read dP^T.
    static constexpr uint32_t DQ_COL = (D == 128) ? DP_COL : 256 + 2 * D;
    static_assert(DQ_COL + D <= TMEM_COLS && DK_COL + D <= TMEM_COLS, "TMEM budget");
    static constexpr int THREADS = 512;
    static constexpr uint32_t REGS_LAUNCH = 128;
    static constexpr uint32_t REGS_SOFTMAX = 184;
    static constexpr uint32_t REGS_DQ = 88;
    static constexpr uint32_t REGS_CTRL = 56;
    static_assert(2 * REGS_SOFTMAX + REGS_DQ + REGS_CTRL == 4 * REGS_LAUNCH,
                  "register split must use exactly the launch allocation");
};

// 3-D tiled reduce-add shared -> global (fp32 add in L2; rows outside the
// tensor are skipped), tracked by the issuing thread's bulk async-groups.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap *map, uint32_t src, int x, int y, int z)
{
    asm volatile("cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
                 " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// Wait until every bulk async-group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---------------------------------------------------------------------------
// 1. delta_i = dO_i . O_i (fp32 over the bf16 values), lse2_i = LSE_i log2(e)
// for rows i < n of every head (0 in the padding rows up to n_pad), and a
// zeroed dQ accumulator. D/8 lanes per row, 8 elements (16 bytes) per lane.
template <int D>
__global__ void __launch_bounds__(256)
    attn_bwd_fused_prep_kernel(const __nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ dout,
                         const float *__restrict__ lse, float *__restrict__ lse2,
                         float *__restrict__ delta, float *__restrict__ dq_acc, int64_t bh_count, int n,
                         int n_pad)
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
        float4 *z = reinterpret_cast<float4 *>(dq_acc + off);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int w = L / 2; w >= 1; w /= 2) acc += __shfl_xor_sync(0xffffffffu, acc, w);
    if (valid && part == 0) {
        delta[row] = real ? acc : 0.f;
        lse2[row] = real ? lse[bh * n + i] * 1.4426950408889634f : 0.f;
    }
}

// ---------------------------------------------------------------------------
// 3. dQ (bf16) = dQ accumulator (fp32, already scaled); 8 elements per thread.
__global__ void __launch_bounds__(256)
    attn_bwd_dq_convert_kernel(const float *__restrict__ dq_acc, __nv_bfloat16 *__restrict__ dq,
                               int64_t count8)
{
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= count8) return;
    const float4 a = reinterpret_cast<const float4 *>(dq_acc)[2 * t];
    const float4 b = reinterpret_cast<const float4 *>(dq_acc)[2 * t + 1];
    uint4 r;
    r.x = pack_bf16x2(a.x, a.y);
    r.y = pack_bf16x2(a.z, a.w);
    r.z = pack_bf16x2(b.x, b.y);
    r.w = pack_bf16x2(b.z, b.w);
    reinterpret_cast<uint4 *>(dq)[t] = r;
}

// ---------------------------------------------------------------------------
// 2. The main backward kernel.
// GENERAL: compiled for grouped-query heads (kv_heads < heads) or the
// block-local mask (block > 0); the other instantiation handles multi-head
// attention under the causal and window masks. NOMASK (never with GENERAL):
// compiled without the mask test, for problems with no mask whose length is
// a whole number of tiles, where no tile needs one; the test sits inside the
// unrolled exponential loop and, never taken there, still cost 3% to 8%.
template <int D, bool GENERAL, bool NOMASK>
__global__ void __launch_bounds__(FusedBwdCfg<D>::THREADS, 1)
    attn_bwd_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                    const __grid_constant__ CUtensorMap tmdQacc, const FusedBwdParams p)
{
    using C = FusedBwdCfg<D>;
    constexpr int NST = C::NST;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    if (base - raw > static_cast<uint32_t>(C::SLACK)) {
        // Cannot happen with a 1 KB-aligned dynamic shared memory base; every
        // thread takes this branch alike, before any barrier or TMEM use.
        if (threadIdx.x == 0) atomicOr(p.status, STATUS_SMEM_ALIGN);
        return;
    }
    uint8_t *const base_ptr = smem_raw + (base - raw);

    const uint32_t sK = base + C::K_OFF, sV = base + C::V_OFF, sDS = base + C::DS_OFF;
    auto sQ = [&](int s) { return base + C::Q_OFF + s * C::TILE_BYTES; };
    auto sdO = [&](int s) { return base + C::DO_OFF + s * C::TILE_BYTES; };
    auto sStat = [&](int s) { return base + C::STAT_OFF + s * 1024; };
    const uint32_t bars = base + C::BAR_OFF;
    const uint32_t kv_full = bars;
    auto q_full = [&](int s) { return bars + 8u * (1 + s); };
    auto q_empty = [&](int s) { return bars + 8u * (1 + NST + s); };
    const uint32_t s_full = bars + 8u * (1 + 2 * NST);
    const uint32_t dp_full = s_full + 8, p_ready = s_full + 16, ds_ready = s_full + 24;
    const uint32_t dq_full = s_full + 32, dq_free = s_full + 40, ds_free = s_full + 48;
    const uint32_t kv_done = s_full + 56, drain_bar = s_full + 64, dqs_free = s_full + 72;
    uint32_t *const tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + C::MISC_OFF);
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(base_ptr + C::MISC_OFF + 4);

    const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x / 32), 0);

    // Work: the key tiles of one head are adjacent in blockIdx (Q / dO reuse
    // in L2); under a causal mask the early key tiles (most query tiles) first.
    // The CTA walks the query tiles [qlo, qhi) of every query head reading
    // this key/value head (grouped-query attention; one head for multi-head
    // attention): item it is query tile qlo + it % nq of the group's head
    // it / nq.
    const int bkv = blockIdx.x / p.num_k_tiles;
    const int G = p.heads / p.kv_heads;
    const int bh0 = (bkv / p.kv_heads) * p.heads + (bkv % p.kv_heads) * G;
    const int kt = static_cast<int>(blockIdx.x % p.num_k_tiles);
    const int k0 = kt * BN;
    const int n = p.n;
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
        mbar_init(dq_full, 1);
        mbar_init(dq_free, BM);
        mbar_init(ds_free, 1);
        mbar_init(kv_done, 1);
        mbar_init(drain_bar, 1);
        mbar_init(dqs_free, 1);
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

    if (warp >= 8 && warp < 12) {
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
        constexpr uint32_t idesc_acc = idesc_bf16_f32(BN, D, 0, 1); // dV, dK: A K-major, B MN-major
        constexpr uint32_t idesc_dq = idesc_bf16_f32(BM, D, 1, 1);  // dQ: A and B MN-major
        bool ok = __all_sync(0xffffffffu, wt.wait(kv_full, 0));
        tc_fence_after();
        const uint64_t k_kmaj = smem_desc_sw128(sK, 16, 1024);
        const uint64_t v_kmaj = smem_desc_sw128(sV, 16, 1024);
        const uint64_t k_mn = smem_desc_sw128(sK, BOX_BYTES, 1024);
        const uint64_t ds_kmaj = smem_desc_sw128(sDS, 16, 1024);
        const uint64_t ds_mn = smem_desc_sw128(sDS, BOX_BYTES, 1024);
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
        //   dV(it), S(it+1), dK(it), dQ(it), dP(it+1).
        // S(it+1) overwrites P(it) in TMEM right behind dV(it), its reader
        // (MMAs complete in issue order), so the softmax warps can start on
        // tile it+1 as soon as they have produced dS(it), while the tensor
        // core runs dK(it) and dQ(it).
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
            if (!(ok = wait(ds_ready, it & 1u))) break;
            if (D == 64 && it > 0 && !(ok = wait(dq_free, (it - 1) & 1u))) break;
            // dK += dS^T Q: dS^T K-major (keys are rows), Q MN-major
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk) {
                const uint64_t off = static_cast<uint64_t>(((kk / 4) * BOX_BYTES + (kk % 4) * 32) >> 4);
                mma_bf16_ss_if(leader, tmem + C::DK_COL, ds_kmaj + off, q_mn + static_cast<uint64_t>(kk * 128),
                               idesc_acc, (it > 0 || kk > 0) ? 1u : 0u);
            }
            // dQ_it = dS K: the same buffer read with queries as rows (MN-major)
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
                mma_bf16_ss_if(leader, tmem + C::DQ_COL, ds_mn + static_cast<uint64_t>(kk * 128),
                               k_mn + static_cast<uint64_t>(kk * 128), idesc_dq, kk > 0 ? 1u : 0u);
            mma_commit_if(leader, dq_full);
            mma_commit_if(leader, ds_free);
            mma_commit_if(leader, q_empty(s));
            if (it + 1 < nitems) {
                // with D = 128, dQ_it sits in dP's columns: the drain must have read it
                if (D == 128 && !(ok = wait(dq_free, it & 1u))) break;
                issue_dp(it + 1);
            }
        }
        if (ok) mma_commit_if(leader, kv_done);
        // Every MMA this warp issued must finish before TMEM is freed.
        mma_commit_if(leader, drain_bar);
        wt.drain(drain_bar, 0);
      }
    } else if (warp >= 12) {
        // ------------------------------------------------------------ dQ drain
        regs_decrease<C::REGS_DQ>();
        const int r = threadIdx.x % BM;  // query row in the tile == TMEM lane
        const bool issuer = (r == 0);
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
        const float sc = p.scale;
        const uint32_t stage = base + C::DQS_OFF;
        // 32 columns of row r (times scale) into staging box b: 16-byte chunk
        // j of the 128-byte row lands at chunk j ^ (r % 8), the 128-byte
        // swizzle the tensor map uses.
        auto stage32 = [&](const uint32_t (&v)[32], int b) {
            const uint32_t rowp = stage + b * (BM * 128) + r * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t chunk = static_cast<uint32_t>(j) ^ static_cast<uint32_t>(r & 7);
                st_shared_v4(rowp + chunk * 16, f2u(u2f(v[4 * j]) * sc), f2u(u2f(v[4 * j + 1]) * sc),
                             f2u(u2f(v[4 * j + 2]) * sc), f2u(u2f(v[4 * j + 3]) * sc));
            }
        };
        for (int it = 0, qi = 0, g = 0; it < nitems; ++it, next_item<GENERAL>(qi, g, nq)) {
            // all four warps take the same decision (they meet at named
            // barriers below)
            if (!named_bar_and(3, BM, wt.wait(dq_full, it & 1u))) break;
            tc_fence_after();
            const int q0 = (qlo + qi) * BM;
            const int bh = bh0 + g;
#pragma unroll 1
            for (int hf = 0; hf < D / 64; ++hf) {
                uint32_t va[32], vb[32];
                tmem_ld32(lane_base + C::DQ_COL + 64 * hf, va);
                tmem_ld32(lane_base + C::DQ_COL + 64 * hf + 32, vb);
                if (hf == D / 64 - 1) {
                    // dQ_i is in registers: its TMEM columns may be reused
                    tc_fence_before();
                    mbar_arrive(dq_free);
                }
                // the previous reduce-add must have read the staging buffer
                if (issuer) tma_store_wait_read0();
                named_bar_sync(3, BM);
                stage32(va, 0);
                stage32(vb, 1);
                fence_proxy_async_smem();
                named_bar_sync(3, BM);
                if (issuer) {
                    tma_reduce_add_3d(&tmdQacc, stage, 64 * hf, q0, bh);
                    tma_reduce_add_3d(&tmdQacc, stage + BM * 128, 64 * hf + 32, q0, bh);
                    tma_store_commit();
                }
            }
            if (C::DQ_IN_DS && issuer) {
                // the staging used the dS buffer: hand it back to the softmax
                tma_store_wait_read0();
                mbar_arrive(dqs_free);
            }
        }
        // every reduce-add must be complete before the kernel ends
        if (issuer) bulk_wait_all();
    } else {
        // ------------------------------------------------------------ softmax / dS
        regs_increase<C::REGS_SOFTMAX>();
        const int h = warp / 4;                 // query columns [64h, 64h + 64)
        const int r = threadIdx.x % BN;         // key row in the tile == TMEM lane
        const int key = k0 + r;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
        const float sc = p.scale_log2;
        const int causal = p.causal, window = p.window;
        // Block mask: bounds that do not change along the query walk.
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
                    // pairs 16*c2 + 2g and 16*c2 + 2g + 1 of the thread's 32
                    float e[4];
                    if ((2 * g) % 16 < ATTN_BWD_EX2_EMU) {
                        ex2_poly_x2(x01.x, x01.y, e[0], e[1]);
                    } else {
                        e[0] = ex2_approx(x01.x);
                        e[1] = ex2_approx(x01.y);
                    }
                    if ((2 * g + 1) % 16 < ATTN_BWD_EX2_EMU) {
                        ex2_poly_x2(x23.x, x23.y, e[2], e[3]);
                    } else {
                        e[2] = ex2_approx(x23.x);
                        e[3] = ex2_approx(x23.y);
                    }
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
                // P^T over this thread's own, already read, S columns
                tmem_st16(lane_base + C::S_COL + 64 * h + 16 * c2, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_ready);

            ok = __all_sync(0xffffffffu, wt.wait(dp_full, it & 1u));
            if (!ok) break;
            if (it > 0) {
                // dK_{i-1} and dQ_{i-1} must have read the dS buffer (and, at
                // D = 128, the dQ drain must have finished staging in it)
                ok = __all_sync(0xffffffffu, wt.wait(C::DQ_IN_DS ? dqs_free : ds_free, (it - 1) & 1u));
                if (!ok) break;
            }
            tc_fence_after();
            const uint32_t row_addr = sDS + h * BOX_BYTES + r * 128;
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
                // dS^T row r, query columns cb .. cb+31 of box h: 16-byte chunks
                // 4*c2 .. 4*c2+3 of the row, 128-byte swizzled
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint32_t chunk = static_cast<uint32_t>(4 * c2 + q4) ^ static_cast<uint32_t>(r & 7);
                    st_shared_v4(row_addr + chunk * 16, pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                }
            }
            fence_proxy_async_smem();
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

}  // namespace attn_sm100
