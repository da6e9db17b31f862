// attn_decode_kernel.cuh - one decode step against rolling key/value caches.
//
// Each sequence b has one query token at position t = pos[b]; its keys and
// values sit in a W-slot rolling cache, position p in slot p mod W, so the
// cache holds positions max(0, t - W + 1) .. t (the rolling buffer of the
// worked example on "Sparse & sub-quadratic attention": a 4,096-position
// cache serving n = 32,768). Softmax is invariant to the order of its terms,
// so the query attends to slots [0, L) with L = min(t + 1, W), in slot order.
// Query head h reads key/value head h / G, G = H / Hkv (grouped-query
// attention, "week17 efficiency attention", MQA / GQA section).
//
// The step reads every cached key and value once and does 4*d FLOPs per
// (query head, key): it is bound by HBM bandwidth, so it runs on the CUDA
// cores and is organised around streaming the caches:
//   attn_decode_kernel: one CTA per (split of the slots, batch * kv head).
//     The CTA's G query rows sit in shared memory (fp32); K and V tiles of 64
//     slots stream in by TMA (128-byte swizzle) through a two-stage ring.
//     Per tile: scores (thread = key; its q rows come as broadcasts), an
//     online softmax per query head (running max and sum), and O += P V
//     (thread = 8 columns of d x a subset of the tile's keys, all G heads).
//     The CTA writes its unnormalised partial O, running max and sum.
//   attn_decode_combine_kernel: merges the splits of every (b, h) with the
//     log-sum-exp rule and writes O (bf16) and LSE.
#pragma once
#include "attn_fwd_kernel.cuh"

namespace attn_sm100 {

constexpr int DEC_TK = 64;         // slots per tile (TMA box rows)
constexpr int DEC_THREADS = 256;
constexpr int DEC_NST = 2;         // K/V ring stages

struct DecodeParams {
    const __nv_bfloat16 *q;  // [B, H, D]
    const int *pos;          // [B], device: position of each sequence's query token
    float *part;             // [nsplit][B*H][D + 2]: unnormalised O, max (log2 units), sum
    int *status;
    int H, Hkv, W;
    int nsplit;
    int chunk;               // slots per split, a multiple of DEC_TK
    float scale_log2;        // scale * log2(e)
};

template <int D, int G>
struct DecCfg {
    static_assert(D == 64 || D == 128, "head size 64 or 128");
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "query heads per key/value head: 1, 2, 4 or 8");
    static constexpr int BOXES = D / BOX_COLS;
    static constexpr int BOX_BYTES_T = DEC_TK * 128;          // one [64 rows x 64 cols] bf16 box
    static constexpr int TILE_BYTES = DEC_TK * D * 2;
    static constexpr int NCH = D / 8;                         // 16-byte chunks per row
    static constexpr int SUBS = DEC_THREADS / NCH;            // key subsets in the P V product
    static constexpr int KPS = DEC_TK / SUBS;                 // keys per subset
    static constexpr int K_OFF = 0;                           // + s * TILE_BYTES
    static constexpr int V_OFF = DEC_NST * TILE_BYTES;        // + s * TILE_BYTES
    static constexpr int Q_OFF = 2 * DEC_NST * TILE_BYTES;    // fp32 [G][D]
    static constexpr int SC_OFF = Q_OFF + G * D * 4;          // fp32 [DEC_TK][G]: scores, then P
    static constexpr int AL_OFF = SC_OFF + DEC_TK * G * 4;    // fp32 [G]: this tile's rescale factors
    static constexpr int BAR_OFF = (AL_OFF + 8 * 4 + 7) / 8 * 8;  // full[NST]
    static constexpr int MISC_OFF = BAR_OFF + DEC_NST * 8;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
    // the end-of-split reduction of the P V partial sums reuses the K/V ring
    static_assert((DEC_THREADS / 32) * G * D * 4 <= 2 * DEC_NST * TILE_BYTES, "reduction buffer");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// bf16 pair (low half first) -> two fp32 values, exactly.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w)
{
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <int D, int G>
__global__ void __launch_bounds__(DEC_THREADS)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const DecodeParams p)
{
    using C = DecCfg<D, G>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - raw);
    float *const q_s = reinterpret_cast<float *>(base_ptr + C::Q_OFF);
    float *const sc = reinterpret_cast<float *>(base_ptr + C::SC_OFF);
    float *const alpha_s = reinterpret_cast<float *>(base_ptr + C::AL_OFF);
    auto sK = [&](int s) { return base + C::K_OFF + s * C::TILE_BYTES; };
    auto sV = [&](int s) { return base + C::V_OFF + s * C::TILE_BYTES; };
    auto full = [&](int s) { return base + C::BAR_OFF + 8u * s; };
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(base_ptr + C::MISC_OFF);

    const int t = threadIdx.x;
    const int split = blockIdx.x;
    const int bkv = blockIdx.y;                 // b * Hkv + kv head
    const int b = bkv / p.Hkv;
    const int h0 = (bkv % p.Hkv) * G;           // first query head of the group
    const int pos = max(p.pos[b], 0);
    const int L = min(pos + 1, p.W);            // valid slots [0, L)
    const int s0 = split * p.chunk;
    const int s1 = min(s0 + p.chunk, L);
    const int ntiles = (s1 > s0) ? (s1 - s0 + DEC_TK - 1) / DEC_TK : 0;
    const size_t prow = static_cast<size_t>(b) * p.H + h0;  // partial row of head h0
    float *const part = p.part + static_cast<size_t>(split) * gridDim.y * G * (D + 2);

    if (ntiles == 0) {
        // no cached slot in this split: an empty partial (max -inf, sum 0)
        for (int i = t; i < G * (D + 2); i += DEC_THREADS) {
            const int g = i / (D + 2), c = i % (D + 2);
            part[(prow + g) * (D + 2) + c] = (c == D) ? -CUDART_INF_F : 0.f;
        }
        return;
    }

    if (t == 0) {
        for (int s = 0; s < DEC_NST; ++s) mbar_init(full(s), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // the group's query rows, fp32
    for (int i = t; i < G * D; i += DEC_THREADS)
        q_s[i] = __bfloat162float(p.q[(static_cast<size_t>(b) * p.H + h0) * D + i]);
    __syncthreads();
    const Waiter wt{abort_flag, p.status};

    auto issue = [&](int tile) {
        const int s = tile % DEC_NST;
        mbar_arrive_expect_tx(full(s), 2 * C::TILE_BYTES);
        const int slot = s0 + tile * DEC_TK;
#pragma unroll
        for (int bx = 0; bx < C::BOXES; ++bx) {
            tma_load_3d(sK(s) + bx * C::BOX_BYTES_T, &tmK, full(s), bx * BOX_COLS, slot, bkv);
            tma_load_3d(sV(s) + bx * C::BOX_BYTES_T, &tmV, full(s), bx * BOX_COLS, slot, bkv);
        }
    };
    int issued = 0;  // tiles whose loads thread 0 has issued
    if (t == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        for (; issued < DEC_NST && issued < ntiles; ++issued) issue(issued);
    }

    // running max (log2 units) and sum of query head g, held by every lane of
    // warp g (warps g >= G leave them unused)
    float m_run = -CUDART_INF_F, l_run = 0.f;
    // P V accumulators: 8 columns [8c, 8c + 8) of every head, over this
    // thread's key subset of each tile
    const int pc = t % C::NCH;
    const int psub = t / C::NCH;
    float acc[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;

    bool ok = true;
    for (int tile = 0; tile < ntiles; ++tile) {
        const int s = tile % DEC_NST;
        ok = __syncthreads_and(wt.wait(full(s), (tile / DEC_NST) & 1u));
        if (!ok) break;
        const int slot0 = s0 + tile * DEC_TK;
        // ---- scores: thread = key k, heads g = gq, gq + 4, ...
        {
            const int k = t % DEC_TK;
            const int gq = t / DEC_TK;
            if (gq < G) {
                constexpr int GPT = (G + 3) / 4;  // heads per thread
                float dot[GPT];
#pragma unroll
                for (int i = 0; i < GPT; ++i) dot[i] = 0.f;
#pragma unroll 4
                for (int j = 0; j < C::NCH; ++j) {
                    const uint32_t addr = sK(s) + (j / 8) * C::BOX_BYTES_T + k * 128 +
                                          ((static_cast<uint32_t>(j % 8) ^ static_cast<uint32_t>(k & 7)) * 16);
                    uint4 kw;
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(kw.x), "=r"(kw.y), "=r"(kw.z), "=r"(kw.w)
                                 : "r"(addr));
                    const float2 k01 = bf16x2_to_f2(kw.x), k23 = bf16x2_to_f2(kw.y);
                    const float2 k45 = bf16x2_to_f2(kw.z), k67 = bf16x2_to_f2(kw.w);
#pragma unroll
                    for (int i = 0; i < GPT; ++i) {
                        const int g = gq + 4 * i;
                        if (g < G) {
                            const float4 qa = *reinterpret_cast<const float4 *>(q_s + g * D + 8 * j);
                            const float4 qb = *reinterpret_cast<const float4 *>(q_s + g * D + 8 * j + 4);
                            float2 d2 = ffma2(k01, make_float2(qa.x, qa.y), make_float2(dot[i], 0.f));
                            d2 = ffma2(k23, make_float2(qa.z, qa.w), d2);
                            d2 = ffma2(k45, make_float2(qb.x, qb.y), d2);
                            d2 = ffma2(k67, make_float2(qb.z, qb.w), d2);
                            dot[i] = d2.x + d2.y;
                        }
                    }
                }
                const bool valid = slot0 + k < s1;
#pragma unroll
                for (int i = 0; i < GPT; ++i) {
                    const int g = gq + 4 * i;
                    if (g < G) sc[k * G + g] = valid ? dot[i] * p.scale_log2 : -CUDART_INF_F;
                }
            }
        }
        __syncthreads();
        // ---- online softmax: warp g handles head g over the tile's keys
        {
            const int w = t / 32, lane = t % 32;
            if (w < G) {
                const float a = sc[lane * G + w], c = sc[(lane + 32) * G + w];
                float mx = fmaxf(a, c);
#pragma unroll
                for (int o = 16; o >= 1; o /= 2) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                const float m_new = fmaxf(m_run, mx);  // finite: the first key of a tile is valid
                const float pa = ex2_approx(a - m_new), pc2 = ex2_approx(c - m_new);
                sc[lane * G + w] = pa;
                sc[(lane + 32) * G + w] = pc2;
                float sum = pa + pc2;
#pragma unroll
                for (int o = 16; o >= 1; o /= 2) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                const float alpha = ex2_approx(m_run - m_new);  // 0 on the first tile
                l_run = l_run * alpha + sum;
                m_run = m_new;
                if (lane == 0) alpha_s[w] = alpha;
            }
        }
        __syncthreads();
        // ---- O += P V over this thread's keys, all heads, columns [8 pc, 8 pc + 8)
        {
            float al[G];
#pragma unroll
            for (int g = 0; g < G; ++g) al[g] = alpha_s[g];
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[g][e] *= al[g];
#pragma unroll
            for (int kk = 0; kk < C::KPS; ++kk) {
                const int k = psub * C::KPS + kk;
                // slots past the cache: P is 0, but the slot may hold NaN
                // (0 * NaN would reach O), so it is skipped
                if (slot0 + k >= s1) continue;
                const uint32_t addr = sV(s) + (pc / 8) * C::BOX_BYTES_T + k * 128 +
                                      ((static_cast<uint32_t>(pc % 8) ^ static_cast<uint32_t>(k & 7)) * 16);
                uint4 vw;
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(vw.x), "=r"(vw.y), "=r"(vw.z), "=r"(vw.w)
                             : "r"(addr));
                const float2 v01 = bf16x2_to_f2(vw.x), v23 = bf16x2_to_f2(vw.y);
                const float2 v45 = bf16x2_to_f2(vw.z), v67 = bf16x2_to_f2(vw.w);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float pw = sc[k * G + g];
                    const float2 p2 = make_float2(pw, pw);
                    float2 r01 = ffma2(v01, p2, make_float2(acc[g][0], acc[g][1]));
                    float2 r23 = ffma2(v23, p2, make_float2(acc[g][2], acc[g][3]));
                    float2 r45 = ffma2(v45, p2, make_float2(acc[g][4], acc[g][5]));
                    float2 r67 = ffma2(v67, p2, make_float2(acc[g][6], acc[g][7]));
                    acc[g][0] = r01.x; acc[g][1] = r01.y; acc[g][2] = r23.x; acc[g][3] = r23.y;
                    acc[g][4] = r45.x; acc[g][5] = r45.y; acc[g][6] = r67.x; acc[g][7] = r67.y;
                }
            }
        }
        // every thread is done with this stage's K and V (and with sc and
        // alpha_s, which the next tile rewrites): refill the stage
        __syncthreads();
        if (t == 0 && issued < ntiles) issue(issued++);
    }
    // copies still in flight must land before the CTA exits
    if (t == 0)
        for (int s = 0; s < DEC_NST; ++s)
            if (issued > s) wt.drain(full(s), ((issued - 1 - s) / DEC_NST) & 1u);
    if (!__syncthreads_and(ok)) return;

    // ---- reduce the P V partial sums over key subsets: lanes t and t ^ NCH
    // share a column chunk within a warp (for D = 128; D = 64 has more
    // subsets per warp), then the warps through shared memory
    float *const red = reinterpret_cast<float *>(base_ptr + C::K_OFF);  // ring is idle now
#pragma unroll
    for (int o = C::NCH; o < 32; o *= 2)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], o);
    const int w = t / 32, lane = t % 32;
    if (lane < C::NCH) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < 8; ++e) red[(w * G + g) * D + 8 * pc + e] = acc[g][e];
    }
    if (w < G && lane == 0) {
        // this split's max and sum of head w
        part[(prow + w) * (D + 2) + D] = m_run;
        part[(prow + w) * (D + 2) + D + 1] = l_run;
    }
    __syncthreads();
    for (int i = t; i < G * D; i += DEC_THREADS) {
        const int g = i / D, c = i % D;
        float s = 0.f;
#pragma unroll
        for (int ww = 0; ww < DEC_THREADS / 32; ++ww) s += red[(ww * G + g) * D + c];
        part[(prow + g) * (D + 2) + c] = s;
    }
}

// Merge the splits of each (b, h): M = max_s m_s, l = sum_s l_s 2^(m_s - M),
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
