// attn_fwd_kernel.cuh - exact softmax attention forward for sm_100a.
//
// One CTA computes two adjacent 128-row query tiles Q_0, Q_1 (256 rows) of
// one (batch, query head); its keys and values come from the key/value head
// of that query head's group (grouped-query attention; one K/V head per
// query head in the multi-head case). For each key/value tile j allowed by
// the mask:
//   S_s = Q_s K_j^T                     (tcgen05 MMA, smem x smem -> TMEM fp32)
//   online softmax on S_s, row by row   (running max m, running normaliser l)
//   O_s += P_s V_j                      (tcgen05 MMA, P from TMEM x V from smem)
// and at the end O_s / l, LSE = m + ln l are written once. This is the
// FlashAttention tile loop with the online softmax ("week17 efficiency
// attention", FlashAttention section; "Efficient Transformers ...", "The
// online softmax trick"): the running output stays unnormalised and is
// divided once, and only the current tile's scores ever live on chip.
//
// Roles (384 threads, 12 warps = 3 warpgroups, one warp of each per SMSP):
//   warps 0-3  softmax for Q_0; warps 4-7 softmax for Q_1. Thread r of a
//              warpgroup owns query row r (= TMEM lane r): it reads its S row,
//              masks boundary tiles, updates (m, l), writes P (bf16) into TMEM,
//              rescales its O row when m grew, and runs the epilogue
//              (O / l -> bf16 -> smem -> TMA store; LSE store).
//   warp 8     MMA issuer (one elected lane) and TMEM owner; in the
//              persistent form it issues Q_0's MMAs and warp 10 Q_1's.
//   warp 9     TMA producer (one elected lane): Q_0, Q_1 once, then K_j, V_j
//              alternately into a ring of NSLOT shared-memory slots.
//   warps 10-11 otherwise idle (they complete the third warpgroup).
// Registers: launched at 168 per thread; the softmax warpgroups raise theirs
// to 232 (a 128-float S row plus its P stay in registers, no spills) and the
// third warpgroup drops to 40: 2*128*232 + 128*40 = 384*168.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256, 256+D),
// O_1 [256+D, 256+2D); P_s over S_s at D = 128, in its own columns at D = 64
// (P_0 [384,448), P_1 [448,512)).
// MMA issue order per key tile j, D = 128: PV_0(j-1), S_0(j), PV_1(j-1),
// S_1(j). tcgen05 MMAs from one thread complete in issue order, so (a) S_s(j)
// overwrites P_s(j-1) only after PV_s(j-1) has read it, and (b) when S_s(j)
// is complete, PV_s(j-1) is too, so the softmax may rescale O_s right away.
// With one CTA per item the softmax hands P_s over in two halves (keys 0..63,
// then 64..127, each announced on its own barrier; O_s is rescaled before the
// first is announced): the MMA warp issues PV_s on the first half while the
// softmax is still computing the second.
// D = 64: S_0(j), S_1(j), PV_0(j-1), PV_1(j-1), S_s(j) waiting only until the
// softmax has read S_s(j-1) into registers; the softmax waits for PV_s(j-1)
// before it overwrites P_s or rescales O_s.
// The exponentials run on the MUFU, and a fixed share of them on the FMA pipe
// as a polynomial (see ex2_poly_x2): on every tile at d = 64, on unmasked
// tiles at d = 128; the share and the form of the row max differ per head
// size (FwdCfg).
// Instantiations: BLOCKMASK = false for the causal and window masks (the
// closed-form bounds), true for the block-local mask (Mask intervals); and
// PERSIST: one CTA per work item (the pair of query tiles above), or one CTA
// per SM walking a static list of work items. The persistent form is for
// short key ranges (narrow windows, short sequences): there a CTA's set-up,
// Q load and epilogue are as long as its key loop, and the persistent CTA
// overlaps them with the neighbouring items' work. Across items the producer
// reloads Q_s once the last S_s MMA of the previous item is done (q_empty),
// the first PV_s of an item waits until the softmax has read the previous
// O_s out (o_free), and the epilogue writes O straight from registers to
// global memory (the Q buffer may already hold the next item's Q). NOMASK:
// compiled without the mask code, for problems with no mask whose length is a
// whole number of key tiles (no tile is ever masked): the masked branches,
// never taken there, otherwise still cost 1% to 4% on unmasked rows.
//
// Every wait is bounded (about one second). On expiry the kernel sets bit 1
// of the device status word, tells the other roles to stop, waits (bounded)
// for its own copies and MMAs in flight, frees TMEM and returns.
#pragma once
#include <cuda_bf16.h>
#include <type_traits>
#include <math_constants.h>

#include "sm100.cuh"

namespace attn_sm100 {

constexpr int BM = 128;                       // query rows per tile (= TMEM lanes)
constexpr int BN = 128;                       // keys per tile
constexpr int QT = 2;                         // query tiles per CTA
constexpr int BOX_COLS = 64;                  // bf16 columns per 128-byte swizzle atom
constexpr int BOX_BYTES = BM * BOX_COLS * 2;  // one [128 x 64] bf16 box: 16 KB
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;
constexpr uint64_t DRAIN_LIMIT_NS = 200000000ull;
constexpr int STATUS_WAIT_TIMEOUT = 1;

// The running max is replaced as soon as a tile raises it, so the largest P
// entry of every row is exactly 1.0 and its bf16 rounding never reaches O. (A
// stale max saves O rescales but puts up to 2^-9 relative error on the
// dominant term: too much for peaked rows.)

// Exponentials computed on the FMA pipe instead of the MUFU unit: out of every
// 16 pairs of a row, ATTN_EX2_EMU_D* pairs use the polynomial (at d = 128
// spread evenly, pair i when i * EMU mod 16 < EMU; at d = 64 the first ones).
// The splits and the row-max form per head size are the fastest measured in
// runs long enough to reach the power cap: at d = 64 more FMA-pipe work
// gains per clock but lowers the clock more.
#ifndef ATTN_EX2_EMU_D64
#define ATTN_EX2_EMU_D64 3
#endif
#ifndef ATTN_EX2_EMU_D128
#define ATTN_EX2_EMU_D128 5
#endif

struct FwdParams {
    __nv_bfloat16 *o;  // [B*H, n, D]: written directly by the persistent form
    float *lse;        // [B*H, n]
    int *status;       // device status word
    int heads;         // H: query heads per batch
    int kv_heads;      // H_kv: key/value heads per batch (divides H)
    int n;
    int num_q_tiles;   // ceil(n / BM)
    int num_cta_tiles; // ceil(num_q_tiles / QT): work items per (batch, head)
    int num_work;      // B * H * num_cta_tiles
    int pair_major;    // persistent form: items pair-major (else head-major)
    float scale_log2;  // scale * log2(e)
    int causal;
    int window;        // < 0: none
    int block;         // > 0: block-local mask with blocks of this many tokens
};

template <int D>
struct FwdCfg {
    static_assert(D == 64 || D == 128, "head size 64 or 128");
    static constexpr int TILE_BYTES = BM * D * 2;    // 128 rows x D bf16
    static constexpr int BOXES = D / BOX_COLS;
    static constexpr int NSLOT = (D == 128) ? 5 : 8;  // K/V ring slots (one tile each)
    static constexpr int Q_OFF = 0;
    static constexpr int KV_OFF = Q_OFF + QT * TILE_BYTES;
    static constexpr int BAR_OFF = KV_OFF + NSLOT * TILE_BYTES;
    // q_full[QT], kv_full[NSLOT], kv_empty[NSLOT], s_full[QT], p_full[QT], o_done[QT],
    // s_free[QT], pv_done[QT], o_free[QT], q_empty[QT], drain[QT], p_half[QT]
    static constexpr int NUM_BARS = 2 * QT + 2 * NSLOT + 8 * QT;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + 1 KB alignment slack
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t S_COL = 0;    // + s * BN
    static constexpr uint32_t O_COL = 256;  // + s * D
    // With D = 64 TMEM has room for P buffers of their own (64 columns of
    // packed bf16 per tile), so S(j+1) can be computed as soon as the softmax
    // has read S(j): the MMA round trip leaves the softmax's critical path.
    // With D = 128 TMEM is full and P overwrites its S.
    static constexpr bool SPLIT_P = (D == 64);
    static constexpr uint32_t P_COL = SPLIT_P ? 256 + QT * D : S_COL;  // + s * (SPLIT_P ? BN/2 : BN)
    static constexpr uint32_t P_STRIDE = SPLIT_P ? BN / 2 : BN;
    static_assert(!SPLIT_P || P_COL + QT * P_STRIDE <= TMEM_COLS, "TMEM budget");
    static constexpr int THREADS = 384;
    static constexpr uint32_t REGS_LAUNCH = 168;   // 65536 / 384, rounded down to 8
    static constexpr uint32_t REGS_SOFTMAX = 232;
    static constexpr uint32_t REGS_OTHER = 40;
    static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_OTHER == THREADS * REGS_LAUNCH,
                  "register split must use exactly the launch allocation");
    static constexpr int EX2_EMU = (D == 128) ? ATTN_EX2_EMU_D128 : ATTN_EX2_EMU_D64;
    static constexpr bool EMU_SPREAD = (D == 128);  // polynomial pairs spread along the row
    static constexpr bool MAX3 = (D == 128);        // row max with three-input max
    // Boundary (masked) tiles take the polynomial share too, their masked
    // entries zeroed in P afterwards: at d = 64 +4% to +5% on causal
    // workloads; at d = 128 the same cost 1% to 4%, so there they use the
    // MUFU alone.
    static constexpr bool EMU_MASKED = (D == 64);
    // D = 128, one CTA per item: P handed over in two halves of 64 keys, the
    // PV MMAs of the first half running while the softmax computes the
    // second (measured +2% to +3%; slower in the persistent form, which
    // keeps one hand-over).
    static constexpr bool PV_SPLIT = (D == 128);
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
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

// Every mask as intervals: query i attends to the keys [first_key(i),
// last_key(i)], key j is attended by the queries [first_query(j),
// last_query(j)]. Masks: causal (j <= i); a window w >= 0 (keys from i - w,
// and up to i + w when not causal); a block-local mask with blocks of b
// tokens (keys of the query's block and of the previous one, and j <= i when
// causal). The host passes w <= n - 2 and b < n (wider ones allow the same
// keys as no such mask) and never a window and a block together. All four
// bounds are non-decreasing in their argument.
struct Mask {
    int n, causal, window, block;

    __device__ __forceinline__ int first_key(int i) const
    {
        if (window >= 0) return max(0, i - window);
        if (block > 0) return max(0, (i / block - 1) * block);
        return 0;
    }
    __device__ __forceinline__ int last_key(int i) const
    {
        int64_t hi = static_cast<int64_t>(n) - 1;
        if (causal)
            hi = i;
        else if (window >= 0)
            hi = static_cast<int64_t>(i) + window;
        else if (block > 0)
            hi = (static_cast<int64_t>(i / block) + 1) * block - 1;
        return static_cast<int>(min(hi, static_cast<int64_t>(n) - 1));
    }
    __device__ __forceinline__ int first_query(int j) const
    {
        if (causal) return j;
        if (window >= 0) return max(0, j - window);
        if (block > 0) return (j / block) * block;
        return 0;
    }
    __device__ __forceinline__ int last_query(int j) const
    {
        int64_t hi = static_cast<int64_t>(n) - 1;
        if (window >= 0)
            hi = static_cast<int64_t>(j) + window;
        else if (block > 0)
            hi = (static_cast<int64_t>(j / block) + 2) * block - 1;
        return static_cast<int>(min(hi, static_cast<int64_t>(n) - 1));
    }
};

// Key tiles [jlo, jhi) holding at least one key allowed for some row of the
// query tile starting at m0 (fully masked tiles are never visited). Empty when
// the query tile lies past n. Causal and window masks only (the kernels'
// specialisation without a block mask keeps this arithmetic).
__device__ __forceinline__ void key_tile_range(int m0, int n, int causal, int window, int &jlo,
                                               int &jhi)
{
    if (m0 >= n) {
        jlo = jhi = 0;
        return;
    }
    int kend = n;  // exclusive
    if (causal)
        kend = min(n, m0 + BM);
    else if (window >= 0)
        kend = min(n, m0 + BM + window);
    const int kbeg = (window >= 0) ? max(0, m0 - window) : 0;
    jlo = kbeg / BN;
    jhi = (kend + BN - 1) / BN;
}

// The same for any Mask (used with a block mask).
__device__ __forceinline__ void key_tile_range(int m0, const Mask &mk, int &jlo, int &jhi)
{
    if (m0 >= mk.n) {
        jlo = jhi = 0;
        return;
    }
    jlo = mk.first_key(m0) / BN;
    jhi = (mk.last_key(min(m0 + BM - 1, mk.n - 1)) + 1 + BN - 1) / BN;
}

__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }
__device__ __forceinline__ uint32_t f2u(float x) { return __float_as_uint(x); }

// 2^x on the FMA pipe for x in [-125, 0.5]: x = k + f with k = round(x) and
// f in [-1/2, 1/2]; 2^f by a degree-3 polynomial (minimax relative error
// 7.5e-5, coefficients fitted by gen_exp2_poly.py), 2^k added to the exponent
// field. Two lanes at a time with packed fp32 instructions.
__device__ __forceinline__ void ex2_poly_x2(float x0, float x1, float &y0, float &y1)
{
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer
    x0 = fmaxf(x0, -125.0f);
    x1 = fmaxf(x1, -125.0f);
    const float2 t = fadd2(make_float2(x0, x1), make_float2(kRound, kRound));
    const float2 r = fsub2(t, make_float2(kRound, kRound));          // round(x)
    const float2 f = fsub2(make_float2(x0, x1), r);
    float2 p = ffma2(make_float2(0.05517167f, 0.05517167f), f, make_float2(0.24261113f, 0.24261113f));
    p = ffma2(p, f, make_float2(0.69326097f, 0.69326097f));
    p = ffma2(p, f, make_float2(0.99992806f, 0.99992806f));
    // t's low mantissa bits hold k (offset by 0x4B400000, whose bits vanish
    // when shifted left by 23): add k << 23 to the exponent of p.
    y0 = u2f(f2u(p.x) + (f2u(t.x) << 23));
    y1 = u2f(f2u(p.y) + (f2u(t.y) << 23));
}

// One work item: two adjacent 128-row query tiles of one (batch, query head),
// their key-tile ranges and the union of those.
struct FwdWork {
    int bh, bkv, m0;
    int jlo_s[QT], jhi_s[QT];
    int jlo, jhi;  // union [jlo, jhi): contiguous; empty tiles have jlo_s == jhi_s
};

// Work item w. Head-major: the query-tile pairs of one head are consecutive
// (K/V reuse in L2) and, within a head, the late pairs (the most expensive
// under a causal mask) come first; one CTA per item then gets the next item
// from the hardware whenever an SM frees up. Pair-major (persistent form,
// causal mask): the late, heaviest pairs of every head first, so that the
// snake order of fwd_item gives every CTA about the same work.
template <bool BLOCKMASK, bool PERSIST>
__device__ __forceinline__ FwdWork fwd_work(const FwdParams &p, int w)
{
    FwdWork t;
    const int bh_count = p.num_work / p.num_cta_tiles;
    const bool pair_major = PERSIST && p.pair_major;
    t.bh = pair_major ? w % bh_count : w / p.num_cta_tiles;
    // Grouped-query attention: query head h of batch b reads key/value head
    // h / (H / H_kv) of that batch (H_kv = H: one K/V head per query head).
    t.bkv = (t.bh / p.heads) * p.kv_heads + (t.bh % p.heads) / (p.heads / p.kv_heads);
    const int ct = p.num_cta_tiles - 1 - (pair_major ? w / bh_count : w % p.num_cta_tiles);
    t.m0 = ct * (QT * BM);
#pragma unroll
    for (int s = 0; s < QT; ++s) {
        if constexpr (BLOCKMASK)
            key_tile_range(t.m0 + s * BM, Mask{p.n, p.causal, p.window, p.block}, t.jlo_s[s], t.jhi_s[s]);
        else
            key_tile_range(t.m0 + s * BM, p.n, p.causal, p.window, t.jlo_s[s], t.jhi_s[s]);
    }
    // Union of the ranges: starts with tile 0's, ends with the last non-empty
    // tile's.
    t.jlo = t.jlo_s[0];
    t.jhi = (t.jhi_s[1] > t.jlo_s[1]) ? max(t.jhi_s[0], t.jhi_s[1]) : t.jhi_s[0];
    return t;
}

// The k-th work item of CTA c (of G = gridDim.x): one per CTA without
// persistence; persistent CTAs take items k*G + c, and with pair-major items
// k*G + G-1-c on odd passes k (a snake over the heavy-first list, so that
// every CTA gets heavy and light items alike); -1 when the last, partial pass
// has none for this CTA, -2 past the end. (Head-major items keep the plain
// round robin: measured 5% to 16% faster than the snake on windowed masks.)
template <bool PERSIST>
__device__ __forceinline__ int fwd_item(const FwdParams &p, int k)
{
    if (!PERSIST) return k == 0 ? static_cast<int>(blockIdx.x) : -2;
    const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    const int64_t first = static_cast<int64_t>(k) * G;
    if (first >= p.num_work) return -2;
    const int64_t w = first + ((p.pair_major && (k & 1)) ? G - 1 - c : c);
    return w < p.num_work ? static_cast<int>(w) : -1;
}

// BLOCKMASK: compiled for the block-local mask (p.block > 0); the other
// instantiation handles the causal and window masks.
// PERSIST: one CTA per SM walks work items blockIdx.x, blockIdx.x + gridDim.x,
// ... (for short key ranges, where a CTA's start-up, Q load and epilogue
// would otherwise not be amortised); else one CTA per work item. Every
// mbarrier phase is counted across items, so both forms run the same code.
// NOMASK: no mask and n a multiple of BN (the host chooses it; never with
// BLOCKMASK).
template <int D, bool BLOCKMASK, bool PERSIST, bool NOMASK>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const FwdParams p)
{
    using C = FwdCfg<D>;
    constexpr int NSLOT = C::NSLOT;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - raw);

    auto sQ = [&](int s) { return base + C::Q_OFF + s * C::TILE_BYTES; };
    auto sKV = [&](int slot) { return base + C::KV_OFF + slot * C::TILE_BYTES; };
    const uint32_t bars = base + C::BAR_OFF;
    auto q_full = [&](int s) { return bars + 8u * s; };
    auto kv_full = [&](int slot) { return bars + 8u * (QT + slot); };
    auto kv_empty = [&](int slot) { return bars + 8u * (QT + NSLOT + slot); };
    auto s_full = [&](int s) { return bars + 8u * (QT + 2 * NSLOT + s); };
    auto p_full = [&](int s) { return bars + 8u * (2 * QT + 2 * NSLOT + s); };
    auto o_done = [&](int s) { return bars + 8u * (3 * QT + 2 * NSLOT + s); };
    auto s_free = [&](int s) { return bars + 8u * (4 * QT + 2 * NSLOT + s); };
    auto pv_done = [&](int s) { return bars + 8u * (5 * QT + 2 * NSLOT + s); };
    auto o_free = [&](int s) { return bars + 8u * (6 * QT + 2 * NSLOT + s); };
    auto q_empty = [&](int s) { return bars + 8u * (7 * QT + 2 * NSLOT + s); };
    auto drain_bar = [&](int s) { return bars + 8u * (8 * QT + 2 * NSLOT + s); };
    auto p_half = [&](int s) { return bars + 8u * (9 * QT + 2 * NSLOT + s); };
    // The persistent form gives each query-tile slot an MMA issuer of its own
    // (warp 8: slot 0, warp 10: slot 1), so that one slot's walk over its key
    // tiles and items never waits for the other's: with a window the two
    // tiles of an item walk key ranges one tile apart, and with one issuer
    // the next item's first S waited for the later tile's last PV.
    constexpr bool DUAL = PERSIST;
    constexpr bool PV_SPLIT = C::PV_SPLIT && !PERSIST;  // single issuer only
    uint32_t *const tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + C::MISC_OFF);
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(base_ptr + C::MISC_OFF + 4);

    // Warp index broadcast from lane 0, so the compiler knows it is uniform
    // across the warp (role branches then keep warp-uniform values in
    // uniform registers).
    const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x / 32), 0);
    const int lane = threadIdx.x % 32;
    const int n = p.n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < QT; ++s) {
            mbar_init(q_full(s), 1);
            mbar_init(s_full(s), 1);
            mbar_init(p_full(s), BM);
            mbar_init(p_half(s), BM);
            mbar_init(o_done(s), 1);
            mbar_init(s_free(s), BM);
            mbar_init(pv_done(s), 1);
            mbar_init(o_free(s), BM);
            mbar_init(q_empty(s), 1);
        }
        for (int i = 0; i < NSLOT; ++i) {
            mbar_init(kv_full(i), 1);
            mbar_init(kv_empty(i), DUAL ? QT : 1);  // one release per issuing warp
        }
        for (int s = 0; s < QT; ++s) mbar_init(drain_bar(s), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        if (!PERSIST) tma_prefetch_desc(&tmO);
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
      // Third warpgroup: TMA producer, MMA issuer and two idle warps.
      regs_decrease<C::REGS_OTHER>();
      const uint32_t leader = elect_one();
      if (warp == 9) {
        // ------------------------------------------------------------ TMA producer
        // The whole warp runs this loop (uniform operands); one lane issues.
        int qn[QT] = {};  // Q loads issued per tile slot
        int item = 0;     // K/V ring items issued: K and V of each key tile
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int w = fwd_item<PERSIST>(p, it);
            if (w == -2) break;
            if (w < 0) continue;
            const FwdWork t = fwd_work<BLOCKMASK, PERSIST>(p, w);
#pragma unroll
            for (int s = 0; s < QT; ++s) {
                if (!ok || t.jhi_s[s] <= t.jlo_s[s]) continue;
                // Q_s is free once the previous item's last S_s MMA is done.
                if (qn[s] > 0 && !__all_sync(0xffffffffu, wt.wait(q_empty(s), (qn[s] - 1) & 1u))) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx_if(leader, q_full(s), C::TILE_BYTES);
#pragma unroll
                for (int b = 0; b < C::BOXES; ++b)
                    tma_load_3d_if(leader, sQ(s) + b * BOX_BYTES, &tmQ, q_full(s), b * BOX_COLS,
                                   t.m0 + s * BM, t.bh);
                ++qn[s];
            }
            // K and V of key tile jlo + i/2 (i even: K, odd: V)
            for (int i = 0; ok && i < 2 * (t.jhi - t.jlo); ++i, ++item) {
                const int slot = item % NSLOT;
#ifdef ATTN_FAULT_DROP_FIRST_V
                // Test hook (never defined in the library build): the V tile of
                // the first key tile is never loaded, so the MMA warp's wait on it
                // must expire and the kernel must stop cleanly.
                if (item == 1) continue;
#endif
                if (item >= NSLOT &&
                    !__all_sync(0xffffffffu, wt.wait(kv_empty(slot), ((item / NSLOT) & 1u) ^ 1u))) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx_if(leader, kv_full(slot), C::TILE_BYTES);
                const CUtensorMap *map = (i & 1) ? &tmV : &tmK;
                const int k0 = (t.jlo + i / 2) * BN;
#pragma unroll
                for (int b = 0; b < C::BOXES; ++b)
                    tma_load_3d_if(leader, sKV(slot) + b * BOX_BYTES, map, kv_full(slot), b * BOX_COLS, k0, t.bkv);
            }
        }
        if (!ok) {
            // Aborted: let every copy issued into shared memory land first.
#pragma unroll
            for (int s = 0; s < QT; ++s)
                if (qn[s] > 0) wt.drain(q_full(s), (qn[s] - 1) & 1u);
            for (int slot = 0; slot < NSLOT; ++slot)
                if (item > slot) wt.drain(kv_full(slot), ((item - 1 - slot) / NSLOT) & 1u);
        }
      } else if (DUAL && (warp == 8 || warp == 10)) {
        // ------------------------------------------------------------ MMA issuers, one per slot
        // Both walk every key tile of every item and release each ring slot
        // (kv_empty counts one release per warp), after waiting for the slot
        // to fill, also when their tile does not use it: so neither can
        // release a slot's next use before the other has released this one.
        const int s = (warp == 10) ? 1 : 0;
        constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, 0, 0);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, 0, 1);
        const uint64_t kdesc0 = smem_desc_sw128(sKV(0), 16, 1024);
        const uint64_t vdesc0 = smem_desc_sw128(sKV(0), BOX_BYTES, 1024);
        const uint32_t s_col = tmem + C::S_COL + s * BN;
        const uint32_t o_col = tmem + C::O_COL + s * D;
        const uint32_t p_col = tmem + C::P_COL + s * C::P_STRIDE;
        int qn = 0, sn = 0, pn = 0, tn = 0;  // Q tiles, S and PV MMAs, items of this slot
        int item = 0;                        // ring items walked
        bool issued = false;                 // any MMA issued by this warp yet
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int w = fwd_item<PERSIST>(p, it);
            if (w == -2) break;
            if (w < 0) continue;
            const FwdWork t = fwd_work<BLOCKMASK, PERSIST>(p, w);
            const int my_lo = s ? t.jlo_s[1] : t.jlo_s[0], my_hi = s ? t.jhi_s[1] : t.jhi_s[0];
            if (my_hi > my_lo) {
                ok = __all_sync(0xffffffffu, wt.wait(q_full(s), qn & 1u));
                ++qn;
            }
            tc_fence_after();
            const uint64_t qdesc = smem_desc_sw128(sQ(s), 16, 1024);
            const int item0 = item;
            for (int j = t.jlo; ok && j <= t.jhi; ++j) {
                const int ik = item0 + 2 * (j - t.jlo);
                const int iv = ik - 1;
                if (j < t.jhi && !__all_sync(0xffffffffu, wt.wait(kv_full(ik % NSLOT), (ik / NSLOT) & 1u))) {
                    ok = false;
                    break;
                }
                if (j > t.jlo && !__all_sync(0xffffffffu, wt.wait(kv_full(iv % NSLOT), (iv / NSLOT) & 1u))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t kdesc = kdesc0 + static_cast<uint64_t>(((ik % NSLOT) * C::TILE_BYTES) >> 4);
                const uint64_t vdesc = vdesc0 + static_cast<uint64_t>(((iv % NSLOT) * C::TILE_BYTES) >> 4);
                auto issue_pv = [&]() -> bool {
                    const bool first = (j - 1 == my_lo);
                    if (!__all_sync(0xffffffffu, wt.wait(p_full(s), pn & 1u))) return false;
                    if (first && tn > 0 && !__all_sync(0xffffffffu, wt.wait(o_free(s), (tn - 1) & 1u)))
                        return false;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < BN / 16; ++k)
                        mma_bf16_ts_if(leader, o_col, p_col + k * 8, vdesc + static_cast<uint64_t>(k * 128),
                                       idesc_pv, (!first || k > 0) ? 1u : 0u);
                    ++pn;
                    if constexpr (C::SPLIT_P) mma_commit_if(leader, pv_done(s));
                    if (j == my_hi) {
                        mma_commit_if(leader, o_done(s));
                        ++tn;
                    }
                    return true;
                };
                auto issue_s = [&]() -> bool {
                    if constexpr (C::SPLIT_P) {
                        if (sn > 0 && !__all_sync(0xffffffffu, wt.wait(s_free(s), (sn - 1) & 1u))) return false;
                        tc_fence_after();
                    }
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint64_t off = static_cast<uint64_t>(((k / 4) * BOX_BYTES + (k % 4) * 32) >> 4);
                        mma_bf16_ss_if(leader, s_col, qdesc + off, kdesc + off, idesc_qk, k > 0 ? 1u : 0u);
                    }
                    mma_commit_if(leader, s_full(s));
                    ++sn;
                    if (j == my_hi - 1) mma_commit_if(leader, q_empty(s));
                    return true;
                };
                const bool use_s = j >= my_lo && j < my_hi;
                const bool use_pv = j - 1 >= my_lo && j - 1 < my_hi;
                if constexpr (C::SPLIT_P) {
                    if (use_s) ok = issue_s();
                    if (ok && use_pv) ok = issue_pv();
                } else {
                    if (use_pv) ok = issue_pv();
                    if (ok && use_s) ok = issue_s();
                }
                if (!ok) break;
                issued = issued || use_s || use_pv;
                // Release the slots once this warp's MMAs reading them are
                // done (a commit tracks every MMA this warp has issued);
                // before its first MMA, a plain arrive.
                if (issued) {
                    if (j < t.jhi) mma_commit_if(leader, kv_empty(ik % NSLOT));
                    if (j > t.jlo) mma_commit_if(leader, kv_empty(iv % NSLOT));
                } else {
                    if (j < t.jhi && leader) mbar_arrive(kv_empty(ik % NSLOT));
                    if (j > t.jlo && leader) mbar_arrive(kv_empty(iv % NSLOT));
                }
            }
            item = item0 + 2 * (t.jhi - t.jlo);
        }
        if (issued) {
            mma_commit_if(leader, drain_bar(s));
            wt.drain(drain_bar(s), 0);
        }
      } else if (!DUAL && warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs this loop (uniform operands); one lane issues
        // every MMA and commit, so the commits track all of its MMAs.
        constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, 0, 0);  // Q, K both K-major
        constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, 0, 1);   // P K-major, V MN-major
        // Descriptors: the start-address field is addr >> 4 in the low 14
        // bits, so adding (byte offset >> 4) moves a descriptor within
        // shared memory (all addresses stay below 2^18).
        const uint64_t kdesc0 = smem_desc_sw128(sKV(0), 16, 1024);
        const uint64_t vdesc0 = smem_desc_sw128(sKV(0), BOX_BYTES, 1024);
        int qn[QT] = {};  // q_full phases consumed
        int sn[QT] = {};  // S MMAs issued (s_full commits)
        int pn[QT] = {};  // PV MMAs issued (p_full waits)
        int tn[QT] = {};  // items finished per tile slot (o_done commits)
        int item = 0;     // K/V ring items consumed
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int w = fwd_item<PERSIST>(p, it);
            if (w == -2) break;
            if (w < 0) continue;
            const FwdWork t = fwd_work<BLOCKMASK, PERSIST>(p, w);
#pragma unroll
            for (int s = 0; s < QT; ++s) {
                if (ok && t.jhi_s[s] > t.jlo_s[s]) {
                    ok = __all_sync(0xffffffffu, wt.wait(q_full(s), qn[s] & 1u));
                    ++qn[s];
                }
            }
            tc_fence_after();
            const int item0 = item;  // ring item of K_{jlo}
            for (int j = t.jlo; ok && j <= t.jhi; ++j) {
                const int ik = item0 + 2 * (j - t.jlo);   // ring item of K_j
                const int iv = ik - 1;                    // ring item of V_{j-1}
                if (j < t.jhi && !__all_sync(0xffffffffu, wt.wait(kv_full(ik % NSLOT), (ik / NSLOT) & 1u))) {
                    ok = false;
                    break;
                }
                if (j > t.jlo && !__all_sync(0xffffffffu, wt.wait(kv_full(iv % NSLOT), (iv / NSLOT) & 1u))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t kdesc = kdesc0 + static_cast<uint64_t>(((ik % NSLOT) * C::TILE_BYTES) >> 4);
                const uint64_t vdesc = vdesc0 + static_cast<uint64_t>(((iv % NSLOT) * C::TILE_BYTES) >> 4);
                // O_s += P_s(j-1) V_{j-1}: BN/16 MMAs of 16 keys each
                auto issue_pv = [&](int s) -> bool {
                    const bool first = (j - 1 == t.jlo_s[s]);
                    if (!__all_sync(0xffffffffu, wt.wait(PV_SPLIT ? p_half(s) : p_full(s), pn[s] & 1u)))
                        return false;
                    // The first PV of an item overwrites O_s: the softmax must
                    // have read the previous item's O_s out.
                    if (first && tn[s] > 0 && !__all_sync(0xffffffffu, wt.wait(o_free(s), (tn[s] - 1) & 1u)))
                        return false;
                    tc_fence_after();
                    const uint32_t o_col = tmem + C::O_COL + s * D;
                    const uint32_t p_col = tmem + C::P_COL + s * C::P_STRIDE;
#pragma unroll
                    for (int k = 0; k < BN / 16; ++k) {
                        // the second half of P_s once the softmax has stored it
                        if (PV_SPLIT && k == BN / 32) {
                            if (!__all_sync(0xffffffffu, wt.wait(p_full(s), pn[s] & 1u))) return false;
                            tc_fence_after();
                        }
                        mma_bf16_ts_if(leader, o_col, p_col + k * 8, vdesc + static_cast<uint64_t>(k * 128),
                                       idesc_pv, (!first || k > 0) ? 1u : 0u);
                    }
                    ++pn[s];
                    if constexpr (C::SPLIT_P) mma_commit_if(leader, pv_done(s));
                    if (j == t.jhi_s[s]) {
                        mma_commit_if(leader, o_done(s));
                        ++tn[s];
                    }
                    return true;
                };
                // S_s(j) = Q_s K_j^T: D/16 MMAs of 16 columns each
                auto issue_s = [&](int s) -> bool {
                    if constexpr (C::SPLIT_P) {
                        // the softmax must have read the previous S_s out of TMEM
                        if (sn[s] > 0 && !__all_sync(0xffffffffu, wt.wait(s_free(s), (sn[s] - 1) & 1u)))
                            return false;
                        tc_fence_after();
                    }
                    const uint32_t s_col = tmem + C::S_COL + s * BN;
                    const uint64_t qdesc = smem_desc_sw128(sQ(s), 16, 1024);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint64_t off = static_cast<uint64_t>(((k / 4) * BOX_BYTES + (k % 4) * 32) >> 4);
                        mma_bf16_ss_if(leader, s_col, qdesc + off, kdesc + off, idesc_qk, k > 0 ? 1u : 0u);
                    }
                    mma_commit_if(leader, s_full(s));
                    ++sn[s];
                    // after the item's last S_s MMA, Q_s may be reloaded
                    if (PERSIST && j == t.jhi_s[s] - 1) mma_commit_if(leader, q_empty(s));
                    return true;
                };
                if constexpr (C::SPLIT_P) {
                    // S_0(j), S_1(j), then PV_0(j-1), PV_1(j-1): S(j) goes out as soon as
                    // S(j-1) has been read, long before P(j-1) is ready.
#pragma unroll
                    for (int s = 0; s < QT; ++s)
                        if (ok && j >= t.jlo_s[s] && j < t.jhi_s[s]) ok = issue_s(s);
#pragma unroll
                    for (int s = 0; s < QT; ++s)
                        if (ok && j - 1 >= t.jlo_s[s] && j - 1 < t.jhi_s[s]) ok = issue_pv(s);
                } else {
                    // PV_0(j-1), S_0(j), PV_1(j-1), S_1(j): S_s(j) overwrites P_s(j-1) in
                    // TMEM, so it must follow PV_s(j-1) (MMAs complete in issue order).
#pragma unroll
                    for (int s = 0; s < QT; ++s) {
                        if (ok && j - 1 >= t.jlo_s[s] && j - 1 < t.jhi_s[s]) ok = issue_pv(s);
                        if (ok && j >= t.jlo_s[s] && j < t.jhi_s[s]) ok = issue_s(s);
                    }
                }
                if (!ok) break;
                if (j < t.jhi) mma_commit_if(leader, kv_empty(ik % NSLOT));
                if (j > t.jlo) mma_commit_if(leader, kv_empty(iv % NSLOT));
            }
            item = item0 + 2 * (t.jhi - t.jlo);
        }
        // Every MMA this warp issued must finish before TMEM is freed.
        mma_commit_if(leader, drain_bar(0));
        wt.drain(drain_bar(0), 0);
      }
    } else {
        // ------------------------------------------------------------ softmax
        regs_increase<C::REGS_SOFTMAX>();
        const int s = warp / 4;              // query tile slot of this warpgroup
        const int r = threadIdx.x % BM;      // row in tile == TMEM lane
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
        const uint32_t s_base = lane_base + C::S_COL + s * BN;
        const uint32_t o_base = lane_base + C::O_COL + s * D;
        const uint32_t p_base = lane_base + C::P_COL + s * C::P_STRIDE;
        const float sc = p.scale_log2;
        const int causal = p.causal, window = p.window;
        int sn = 0;  // S tiles consumed (s_full waits) over all items
        int tn = 0;  // items finished (o_done waits)
        bool ok = true;

        for (int it = 0; ok; ++it) {
            const int w = fwd_item<PERSIST>(p, it);
            if (w == -2) break;
            if (w < 0) continue;
            const FwdWork t = fwd_work<BLOCKMASK, PERSIST>(p, w);
            // (selects, not a runtime index: the ranges stay in registers)
            const int my_jlo = s ? t.jlo_s[1] : t.jlo_s[0], my_jhi = s ? t.jhi_s[1] : t.jhi_s[0];
            if (my_jhi <= my_jlo) continue;
            const int q0 = t.m0 + s * BM;    // first row of the tile
            const int row = q0 + r;
            // Block mask: bounds that do not change along the key walk (this
            // row's allowed keys, and the bounds every row of the tile shares).
            const Mask mk{n, p.causal, p.window, p.block};
            const int row_first = mk.first_key(row), row_last = mk.last_key(row);
            const int tile_first = mk.first_key(q0 + BM - 1), tile_last = mk.last_key(q0);
            const int sn0 = sn;              // PV MMAs of this slot before this item
            float mx = -CUDART_INF_F;        // running max, log2 units
            float l = 0.f;                   // running normaliser relative to mx

            for (int j = my_jlo; j < my_jhi; ++j) {
                const int u = j - my_jlo;
                ok = __all_sync(0xffffffffu, wt.wait(s_full(s), sn & 1u));
                if (!ok) break;
                ++sn;
                tc_fence_after();
                uint32_t sv[BN];
                tmem_ld128(s_base, sv);
                if constexpr (C::SPLIT_P) {
                    // S_s is in registers: the MMA warp may overwrite it with S_s(j+1).
                    tc_fence_before();
                    mbar_arrive(s_free(s));
                }

                const int k0 = j * BN;
                // Does some row of the tile lose keys at the top of this key
                // tile (diagonal, ragged end, right edge of a window), or at
                // the bottom (left edge of a window or block)?
                const bool mask_hi =
                    BLOCKMASK ? ((k0 + BN > n) || tile_last < k0 + BN - 1)
                              : ((k0 + BN > n) || (causal && k0 + BN - 1 > q0) ||
                                 (!causal && window >= 0 && k0 + BN - 1 > q0 + window));
                const bool mask_lo = BLOCKMASK ? (tile_first > k0) : (window >= 0 && k0 < q0 + BM - 1 - window);
                const bool need_mask = !NOMASK && (mask_hi || mask_lo);
                // Allowed keys of this row form one interval; in tile columns:
                // [lo, hi] with key = k0 + column (on a side that cuts no row,
                // the bound lies outside the tile). At d = 64 computed up
                // front (the zeroing after the exponentials needs them too),
                // at d = 128 inside the masked branch: 1% faster each.
                auto col_hi = [&]() {
                    return BLOCKMASK ? row_last - k0
                                     : min(causal ? row - k0 : (window >= 0 ? row + window - k0 : BN - 1),
                                           n - 1 - k0);
                };
                auto col_lo = [&]() {
                    return BLOCKMASK ? row_first - k0 : ((window >= 0) ? row - window - k0 : 0);
                };
                int hi = 0, lo = 0;
                if constexpr (C::EMU_MASKED) {
                    hi = col_hi();
                    lo = col_lo();
                }
                if (need_mask) {
                    // Most masked tiles cut on one side only, which takes one
                    // compare per element.
                    if constexpr (!C::EMU_MASKED) {
                        hi = col_hi();
                        lo = col_lo();
                    }
                    if (mask_hi && mask_lo) {
#pragma unroll
                        for (int c = 0; c < BN; ++c)
                            if (c > hi || c < lo) sv[c] = f2u(-CUDART_INF_F);
                    } else if (mask_hi) {
#pragma unroll
                        for (int c = 0; c < BN; ++c)
                            if (c > hi) sv[c] = f2u(-CUDART_INF_F);
                    } else {
#pragma unroll
                        for (int c = 0; c < BN; ++c)
                            if (c < lo) sv[c] = f2u(-CUDART_INF_F);
                    }
                }
                // row max: eight running maxima, of three-input max instructions
                // at d = 128 and of two-input ones at d = 64 (the faster form of
                // each under the power cap)
                float pm[8];
                if constexpr (C::MAX3) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) pm[i] = fmax3(u2f(sv[i]), u2f(sv[8 + i]), u2f(sv[16 + i]));
#pragma unroll
                    for (int c = 24; c + 16 <= BN; c += 16)
#pragma unroll
                        for (int i = 0; i < 8; ++i) pm[i] = fmax3(pm[i], u2f(sv[c + i]), u2f(sv[c + 8 + i]));
#pragma unroll
                    for (int i = 0; i < 8; ++i) pm[i] = fmaxf(pm[i], u2f(sv[BN - 8 + i]));
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) pm[i] = fmaxf(u2f(sv[i]), u2f(sv[8 + i]));
#pragma unroll
                    for (int c = 16; c < BN; c += 8)
#pragma unroll
                        for (int i = 0; i < 8; ++i) pm[i] = fmaxf(pm[i], u2f(sv[c + i]));
                }
                const float tmax = C::MAX3 ? fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]))
                                           : fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                                   fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
                const float mnew = fmaxf(mx, tmax * sc);
                const bool rescale = mnew > mx;
                // alpha = 2^(m_old - m_new): 1 when the max did not grow, 0 when
                // m_old = -inf; the selects avoid (-inf) - (-inf) and a branch.
                const bool none_yet = (mnew == -CUDART_INF_F);
                const float alpha = none_yet ? 1.f : ex2_approx(mx - mnew);
                mx = mnew;
                const float off = none_yet ? 0.f : mx;
                const float2 sc2 = make_float2(sc, sc);
                const float2 noff2 = make_float2(-off, -off);
                float2 ps[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) ps[i] = make_float2(0.f, 0.f);
                uint32_t pk[BN / 2];
                // One straight-line body per case (no branch inside the unrolled
                // loop, so MUFU and FMA work can be interleaved freely). At
                // d = 128 masked tiles use the MUFU alone.
                auto exps = [&](auto emu, auto i0, auto i1) {
                    constexpr int EMU = decltype(emu)::value;
#pragma unroll
                    for (int i = decltype(i0)::value; i < decltype(i1)::value; ++i) {
                        const float2 x = ffma2(make_float2(u2f(sv[2 * i]), u2f(sv[2 * i + 1])), sc2, noff2);
                        float e0, e1;
                        if constexpr (EMU > 0) {
                            // EMU of every 16 pairs: spread evenly along the
                            // row, or the first EMU of each 16
                            if ((C::EMU_SPREAD ? ((i * EMU) % 16) : (i % 16)) < EMU) {
                                ex2_poly_x2(x.x, x.y, e0, e1);
                            } else {
                                e0 = ex2_approx(x.x);
                                e1 = ex2_approx(x.y);
                            }
                        } else {
                            e0 = ex2_approx(x.x);
                            e1 = ex2_approx(x.y);
                        }
                        ps[i & 3] = fadd2(ps[i & 3], make_float2(e0, e1));
                        pk[i] = pack_bf16x2(e0, e1);
                    }
                };
                using I0 = std::integral_constant<int, 0>;
                using IH = std::integral_constant<int, BN / 4>;
                using IE = std::integral_constant<int, BN / 2>;
                const bool emu_off = (C::EX2_EMU == 0) || (!C::EMU_MASKED && need_mask);
                // The polynomial clamps at 2^-125: on masked tiles the masked
                // entries of its pairs are set to exactly 0 in P afterwards
                // (the MUFU gives 0 for them by itself), so a masked key never
                // reaches O, whatever its value. Their 2^-125 stays in the row
                // sum l, below its rounding: from the first allowed key on, l
                // holds the row maximum's 1.0 (and a tile with no allowed key
                // before that is scaled away by alpha = 0).
                auto fix_masked = [&](auto i0, auto i1) {
                    if constexpr (C::EMU_MASKED && C::EX2_EMU > 0) {
#pragma unroll
                        for (int i = decltype(i0)::value; i < decltype(i1)::value; ++i) {
                            if ((C::EMU_SPREAD ? ((i * C::EX2_EMU) % 16) : (i % 16)) < C::EX2_EMU) {
                                const bool k0 = (2 * i >= lo) && (2 * i <= hi);
                                const bool k1 = (2 * i + 1 >= lo) && (2 * i + 1 <= hi);
                                pk[i] &= (k0 ? 0x0000FFFFu : 0u) | (k1 ? 0xFFFF0000u : 0u);
                            }
                        }
                    }
                };
                const bool do_rescale = u > 0 && __any_sync(0xffffffffu, rescale);
                if constexpr (PV_SPLIT) {
                    // First half of P (keys 0..63) -> TMEM; O_s rescaled; the
                    // MMA warp may then run PV on that half while the second
                    // half is computed.
                    if (emu_off)
                        exps(I0{}, I0{}, IH{});
                    else
                        exps(std::integral_constant<int, C::EX2_EMU>{}, I0{}, IH{});
                    if (need_mask) fix_masked(I0{}, IH{});
                    tmem_st32(p_base, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
                    // O_s holds sum_{t<j} P_t V_t (PV_s(j-1) was issued before
                    // S_s(j) and completed with it): rescale when a row's max grew.
                    if (do_rescale) {
                        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
                        for (int h = 0; h < D / 64; ++h) {
                            uint32_t o[64];
                            tmem_ld64(o_base + h * 64, o);
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                const float2 v = fmul2(make_float2(u2f(o[2 * i]), u2f(o[2 * i + 1])), a2);
                                o[2 * i] = f2u(v.x);
                                o[2 * i + 1] = f2u(v.y);
                            }
                            tmem_st64(o_base + h * 64, o);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(p_half(s));
                    if (emu_off)
                        exps(I0{}, IH{}, IE{});
                    else
                        exps(std::integral_constant<int, C::EX2_EMU>{}, IH{}, IE{});
                    if (need_mask) fix_masked(IH{}, IE{});
                    tmem_st32(p_base + BN / 4, *reinterpret_cast<uint32_t(*)[32]>(&pk[BN / 4]));
                    const float2 ps01 = fadd2(ps[0], ps[1]);
                    const float2 ps23 = fadd2(ps[2], ps[3]);
                    const float2 pst = fadd2(ps01, ps23);
                    l = fmaf(l, alpha, pst.x + pst.y);
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(p_full(s));
                    continue;
                }
                if (emu_off)
                    exps(I0{}, I0{}, IE{});
                else
                    exps(std::integral_constant<int, C::EX2_EMU>{}, I0{}, IE{});
                if (need_mask) fix_masked(I0{}, IE{});
                if constexpr (C::SPLIT_P) {
                    // P_s(j) reuses P_s(j-1)'s columns and O_s is about to be
                    // rescaled: PV_s(j-1) must be complete. (The first step of
                    // an item follows the previous item's last PV, which the
                    // epilogue waited for.)
                    if (u > 0) {
                        ok = __all_sync(0xffffffffu, wt.wait(pv_done(s), (sn0 + u - 1) & 1u));
                        if (!ok) break;
                        tc_fence_after();
                    }
                }
                tmem_st64(p_base, pk);
                const float2 ps01 = fadd2(ps[0], ps[1]);
                const float2 ps23 = fadd2(ps[2], ps[3]);
                const float2 pst = fadd2(ps01, ps23);
                l = fmaf(l, alpha, pst.x + pst.y);

                // O_s holds sum_{t<j} P_t V_t: PV_s(j-1) has completed (waited for
                // above with separate P buffers; otherwise it was issued before
                // S_s(j) and completed with it). Rescale when a row's max grew.
                if (do_rescale) {
                    const float2 a2 = make_float2(alpha, alpha);
                    uint32_t o[D];
                    if constexpr (D == 128) tmem_ld128(o_base, o); else tmem_ld64(o_base, o);
#pragma unroll
                    for (int i = 0; i < D / 2; ++i) {
                        const float2 v = fmul2(make_float2(u2f(o[2 * i]), u2f(o[2 * i + 1])), a2);
                        o[2 * i] = f2u(v.x);
                        o[2 * i + 1] = f2u(v.y);
                    }
                    if constexpr (D == 128) tmem_st128(o_base, o); else tmem_st64(o_base, o);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(p_full(s));
            }
            if (ok) ok = __all_sync(0xffffffffu, wt.wait(o_done(s), tn & 1u));
            // Agree before touching O: every warp of the warpgroup goes on or stops.
            ok = named_bar_and(1 + s, BM, ok);
            if (!ok) break;
            ++tn;
            tc_fence_after();
            const float inv_l = 1.f / l;
            if constexpr (PERSIST) {
                // Epilogue: O / l -> bf16, each thread its own row straight
                // to global memory (16-byte stores; rows past n skipped). The
                // Q buffer cannot stage it: the next item's Q may already be
                // loading into it.
                // 64 columns at a time; O_s is free for the next item's first
                // PV once all D columns have been read.
                uint4 *const orow = reinterpret_cast<uint4 *>(p.o + (static_cast<size_t>(t.bh) * n + row) * D);
#pragma unroll
                for (int h = 0; h < D / 64; ++h) {
                    uint32_t o[64];
                    tmem_ld64(o_base + h * 64, o);
                    if (h == D / 64 - 1) {
                        tc_fence_before();
                        mbar_arrive(o_free(s));
                    }
                    if (row < n) {
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            orow[8 * h + c] =
                                make_uint4(pack_bf16x2(u2f(o[8 * c]) * inv_l, u2f(o[8 * c + 1]) * inv_l),
                                           pack_bf16x2(u2f(o[8 * c + 2]) * inv_l, u2f(o[8 * c + 3]) * inv_l),
                                           pack_bf16x2(u2f(o[8 * c + 4]) * inv_l, u2f(o[8 * c + 5]) * inv_l),
                                           pack_bf16x2(u2f(o[8 * c + 6]) * inv_l, u2f(o[8 * c + 7]) * inv_l));
                    }
                }
            } else {
                // Epilogue: O / l -> bf16 -> swizzled smem (this tile's Q buffer,
                // free once its last MMA is done) -> TMA store; rows past n are
                // clipped by the store.
                const uint32_t stage = sQ(s);
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t o[32];
                    tmem_ld32(o_base + c, o);
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack_bf16x2(u2f(o[2 * i]) * inv_l, u2f(o[2 * i + 1]) * inv_l);
                    const uint32_t rowp = stage + (c / BOX_COLS) * BOX_BYTES + r * 128;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t chunk = ((c % BOX_COLS) / 8 + q) ^ (r & 7);
                        st_shared_v4(rowp + chunk * 16, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                    }
                }
                fence_proxy_async_smem();
                named_bar_sync(1 + s, BM);
                if (r == 0) {
                    for (int b = 0; b < C::BOXES; ++b)
                        tma_store_3d(&tmO, stage + b * BOX_BYTES, b * BOX_COLS, q0, t.bh);
                    tma_store_commit();
                    tma_store_wait_read0();
                }
            }
            if (row < n)
                p.lse[static_cast<size_t>(t.bh) * n + row] = (mx + __log2f(l)) * 0.69314718055994531f;
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
