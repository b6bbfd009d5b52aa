// Decode: one new query token per sequence against cached keys, values and
// proxy keys (the inference side of MSA: page "Flash-MSA: Open-Source Sparse
// Attention Kernels Debut", section "How MSA works" -- the Index Branch picks
// KV blocks by max-pooled proxy scores and the Main Branch attends only to
// them; the MiniMax inference kernels the ai-beat post mentions are not
// public, so this path is our own).
//
// The token of sequence b sits at position i = lens[b] - 1 of its caches (its
// own key, value and proxy key are already stored there).  Four kernels:
//   1. proxy scores of the token against keys 0..i, max-pooled per 128-key
//      block (coalesced scan of the proxy-key cache; HBM bound);
//   2. per (b, group): forced blocks plus the best topk - nf others, ranked by
//      a shared-memory bitonic sort of (score, id) keys -- the same order as
//      the training path (higher score first, ties to the lower id);
//   3. attention of the G heads over the selected blocks, split over CTAs by
//      blocks (partial max, sum and output per split; HBM bound on K/V);
//   4. combine of the splits into O (bf16) and the natural-log L.
// Work per token is tiny and irregular, so CUDA cores do the arithmetic; the
// bytes moved (proxy-key scan, selected K/V tiles) set the time.
#include <math.h>

#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr float kLog2eD = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

MSA_DEV int seq_len(const int32_t* lens, int b, int T) { return lens ? lens[b] : T; }

// ---------------------------------------------------------------- 1. pool
// grid (ceil(nblk / 8), B*Hp), 256 threads: warp w scores key block
// blockIdx.x*8 + w.  Eight lanes share a key row (16 bytes each), so a warp
// reads four whole rows per instruction.  A bad length is flagged in status
// word 1 and the sequence is skipped by every kernel.
__global__ void __launch_bounds__(256) decode_pool_kernel(const __nv_bfloat16* __restrict__ qp,
                                                          const __nv_bfloat16* __restrict__ kp,
                                                          const int32_t* __restrict__ lens, int T, int Hp,
                                                          int dp, float* __restrict__ pooled, int nblk,
                                                          uint32_t* status)
{
    const int bg = blockIdx.y, b = bg / Hp, g = bg % Hp;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int len = seq_len(lens, b, T);
    if (len < 1 || len > T) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status + 1, 1u);
        return;
    }
    const int i = len - 1, bi = i >> 7;
    const int n = blockIdx.x * 8 + warp;
    if (n > bi) return;
    const int sub = lane & 7, r4 = lane >> 3;   // 16-byte chunk of the row, row within the group of 4
    const bool has = sub * 8 < dp;
    float qf[8];
    {
        uint4 u = make_uint4(0, 0, 0, 0);
        if (has) u = *reinterpret_cast<const uint4*>(qp + ((int64_t)b * Hp + g) * dp + sub * 8);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h2[e]);
            qf[2 * e] = f.x;
            qf[2 * e + 1] = f.y;
        }
    }
    // eight row loads in flight per lane before any arithmetic
    float mx = -INFINITY;
#pragma unroll 1
    for (int it0 = 0; it0 < 32; it0 += 8) {
        uint4 u[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int j = n * 128 + (it0 + e) * 4 + r4;
            u[e] = (has && j <= i)
                       ? *reinterpret_cast<const uint4*>(kp + (((int64_t)b * T + j) * Hp + g) * dp + sub * 8)
                       : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int j = n * 128 + (it0 + e) * 4 + r4;
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u[e]);
            float sv = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float2 f = __bfloat1622float2(h2[c]);
                sv = fmaf(qf[2 * c], f.x, sv);
                sv = fmaf(qf[2 * c + 1], f.y, sv);
            }
            sv += __shfl_xor_sync(0xffffffffu, sv, 1);
            sv += __shfl_xor_sync(0xffffffffu, sv, 2);
            sv += __shfl_xor_sync(0xffffffffu, sv, 4);
            if (j <= i) mx = fmaxf(mx, sv);
        }
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (lane == 0) pooled[(int64_t)bg * nblk + n] = mx;
}

// ---------------------------------------------------------------- 2. select
// 64-bit key: larger = ranked first.  High word: the score's bits mapped to an
// unsigned order (-0 counted as +0); low word: the complement of the id, so
// equal scores put the lower id first.  0 marks "not a candidate".
MSA_DEV uint64_t rank_key(float s, int n)
{
    uint32_t u = s == 0.f ? 0u : __float_as_uint(s);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((uint64_t)u << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)n);
}

// In-place bitonic sort of n (a power of two) keys in shared memory by the
// whole CTA, descending.
MSA_DEV void cta_sort_desc(uint64_t* a, int n)
{
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int x = threadIdx.x; x < n; x += blockDim.x) {
                const int y = x ^ j;
                if (y > x) {
                    const bool desc = (x & k) == 0;   // descending segment
                    const uint64_t ax = a[x], ay = a[y];
                    if ((ax < ay) == desc) { a[x] = ay; a[y] = ax; }
                }
            }
            __syncthreads();
        }
    }
}

// grid (B*Hp), 1024 threads; dynamic smem: npad keys (npad = the power of two
// >= nblk, at least topk).
__global__ void __launch_bounds__(1024) decode_select_kernel(const float* __restrict__ pooled,
                                                             const int32_t* __restrict__ lens, int T, int Hp,
                                                             int nblk, int npad, int topk, int window,
                                                             int dilation, int32_t* __restrict__ idx,
                                                             int32_t* __restrict__ nsel)
{
    extern __shared__ uint64_t keys[];
    const int bg = blockIdx.x, b = bg / Hp;
    int32_t* out = idx + (int64_t)bg * topk;
    const int len = seq_len(lens, b, T);
    if (len < 1 || len > T) {   // flagged by the pool kernel; leave an empty selection
        for (int s = threadIdx.x; s < topk; s += blockDim.x) out[s] = -1;
        if (threadIdx.x == 0) nsel[bg] = 0;
        return;
    }
    const int bi = (len - 1) >> 7;
    if (bi + 1 <= topk) {   // every eligible block
        for (int s = threadIdx.x; s < topk; s += blockDim.x) out[s] = s <= bi ? s : -1;
        if (threadIdx.x == 0) nsel[bg] = bi + 1;
        return;
    }
    const int nf = min(window, bi / dilation + 1);   // forced: bi, bi - dilation, ...
    const int kk = topk - nf;
    const float* pr = pooled + (int64_t)bg * nblk;
    for (int n = threadIdx.x; n < npad; n += blockDim.x) {
        const int back = bi - n;
        const bool forced = back >= 0 && back % dilation == 0 && back / dilation < nf;
        keys[n] = (n <= bi && !forced) ? rank_key(pr[n], n) : 0ull;
    }
    __syncthreads();
    cta_sort_desc(keys, npad);
    // the kk best free blocks, then the forced ones, as ids; ascending order
    uint64_t* ids = keys + npad;   // topk slots, padded to a power of two below
    int tp = 1;
    while (tp < topk) tp <<= 1;
    for (int s = threadIdx.x; s < tp; s += blockDim.x) {
        uint64_t v;
        if (s < kk) v = 0xFFFFFFFFull - (keys[s] & 0xFFFFFFFFull);
        else if (s < topk) v = (uint64_t)(bi - (s - kk) * dilation);
        else v = 0xFFFFFFFFFFFFFFFFull;
        ids[s] = ~v;   // descending sort of ~id = ascending ids
    }
    __syncthreads();
    cta_sort_desc(ids, tp);
    for (int s = threadIdx.x; s < topk; s += blockDim.x) out[s] = (int32_t)(~ids[s]);
    if (threadIdx.x == 0) nsel[bg] = topk;
}

// ---------------------------------------------------------------- 3. attention
// grid (S, B*Hkv), 128 threads: split s takes the row's s-th selected block
// (one block per CTA keeps many K/V tiles in flight).  Scores in the base-2
// domain (q pre-scaled by scale*log2e); partial (o, m, l) per head.
constexpr int kSplitBlocks = 1;

template <int D, int G>
struct DecSmem {
    static constexpr int kStride = D + 8;   // bf16 elements per staged row: an odd number of 16-byte units
    static constexpr size_t kTile = 128 * kStride * 2;
    static constexpr size_t kK = 0, kV = kTile;
    static constexpr size_t kQ = 2 * kTile;              // [G][D] fp32
    static constexpr size_t kP = kQ + G * D * 4;         // [G][128] fp32
    static constexpr size_t kRed = kP + G * 128 * 4;     // [2][G][4] fp32: maxima, sums
    static constexpr size_t kTotal = kRed + 2 * G * 4 * 4;
};

template <int D, int G>
__global__ void __launch_bounds__(128) decode_attn_kernel(const __nv_bfloat16* __restrict__ q,
                                                          const __nv_bfloat16* __restrict__ k,
                                                          const __nv_bfloat16* __restrict__ v,
                                                          const int32_t* __restrict__ lens,
                                                          const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ nsel, int T, int Hq,
                                                          int Hkv, int topk, float c1, float* __restrict__ part,
                                                          int S)
{
    using SM = DecSmem<D, G>;
    extern __shared__ __align__(16) uint8_t smem[];
    __nv_bfloat16* ks = (__nv_bfloat16*)(smem + SM::kK);
    __nv_bfloat16* vs = (__nv_bfloat16*)(smem + SM::kV);
    float* qs = (float*)(smem + SM::kQ);
    float* ps = (float*)(smem + SM::kP);
    float* rmax = (float*)(smem + SM::kRed);
    float* rsum = rmax + G * 4;
    const int s = blockIdx.x, bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    float* pm = part + ((int64_t)bg * S + s) * G * (D + 2);   // [G][D + 2]: o, then m, l
    const int len = seq_len(lens, b, T);
    const int ns = (len >= 1 && len <= T) ? nsel[bg] : 0;
    const int i = len - 1;
    if (s >= ns) {   // nothing selected for this split: an empty partial
        for (int x = t; x < G * (D + 2); x += 128) {
            const int c = x % (D + 2);
            pm[x] = c == D ? -INFINITY : 0.f;
        }
        return;
    }
    const int n = idx[(int64_t)bg * topk + s];
    // stage K and V rows of block n (16-byte pieces) as two copy groups, and
    // the G query rows: the scores need only K, so V is still arriving while
    // they are computed
    constexpr int kPieces = D / 8;
    for (int half = 0; half < 2; ++half) {
        const __nv_bfloat16* src = half == 0 ? k : v;
        __nv_bfloat16* dst = half == 0 ? ks : vs;
        for (int x = t; x < 128 * kPieces; x += 128) {
            const int row = x / kPieces, c = x % kPieces;
            const int j = n * 128 + row;
            const bool ok = j <= i;
            const int64_t off = (((int64_t)b * T + (ok ? j : 0)) * Hkv + g) * D + c * 8;
            cp_async_16(smem_u32(dst + row * SM::kStride + c * 8), src + off, ok ? 16u : 0u);
        }
        cp_async_commit();
    }
    for (int x = t; x < G * D; x += 128)
        qs[x] = __bfloat162float(q[((int64_t)b * Hq + g * G) * D + x]) * c1;
    cp_async_wait<1>();   // this thread's K pieces have landed
    __syncthreads();
    // scores: thread t = key t of the block; K 16 bytes and q 16 bytes at a time
    const int j = n * 128 + t;
    const bool valid = j <= i;
    float sc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) sc[h] = 0.f;
    const uint4* kr = reinterpret_cast<const uint4*>(ks + t * SM::kStride);
    const float4* q4 = reinterpret_cast<const float4*>(qs);
#pragma unroll 4
    for (int e8 = 0; e8 < D / 8; ++e8) {
        const uint4 u = kr[e8];
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
        float kf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h2[e]);
            kf[2 * e] = f.x;
            kf[2 * e + 1] = f.y;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float4 a = q4[h * (D / 4) + 2 * e8], c = q4[h * (D / 4) + 2 * e8 + 1];
            sc[h] = fmaf(a.x, kf[0], fmaf(a.y, kf[1], fmaf(a.z, kf[2], fmaf(a.w, kf[3], sc[h]))));
            sc[h] = fmaf(c.x, kf[4], fmaf(c.y, kf[5], fmaf(c.z, kf[6], fmaf(c.w, kf[7], sc[h]))));
        }
    }
    // per head: block max, p = exp2(s - m), block sum
    float m[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float bm = valid ? sc[h] : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
        if (lane == 0) rmax[h * 4 + warp] = bm;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = fmaxf(fmaxf(rmax[h * 4], rmax[h * 4 + 1]), fmaxf(rmax[h * 4 + 2], rmax[h * 4 + 3]));
        const float pv = valid ? ex2_approx(sc[h] - m[h]) : 0.f;
        ps[h * 128 + t] = pv;
        float bs = pv;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bs += __shfl_xor_sync(0xffffffffu, bs, o);
        if (lane == 0) rsum[h * 4 + warp] = bs;
    }
    cp_async_wait<0>();   // and the V pieces
    __syncthreads();
    // PV: thread t = head-dim index; P four keys at a time
    if (t < D) {
        float acc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = 0.f;
        const float4* p4 = reinterpret_cast<const float4*>(ps);
#pragma unroll 2
        for (int k4 = 0; k4 < 32; ++k4) {
            float vf[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) vf[e] = __bfloat162float(vs[(4 * k4 + e) * SM::kStride + t]);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float4 pp = p4[h * 32 + k4];
                acc[h] = fmaf(pp.x, vf[0], fmaf(pp.y, vf[1], fmaf(pp.z, vf[2], fmaf(pp.w, vf[3], acc[h]))));
            }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) pm[h * (D + 2) + t] = acc[h];
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
        if (t == h) {
            pm[h * (D + 2) + D] = m[h];
            pm[h * (D + 2) + D + 1] = rsum[h * 4] + rsum[h * 4 + 1] + rsum[h * 4 + 2] + rsum[h * 4 + 3];
        }
}

// ---------------------------------------------------------------- 4. combine
// grid (B*Hq), D threads: O = sum_s 2^(m_s - M) o_s / L, L = sum_s 2^(m_s - M) l_s;
// lse = (M + log2 L) ln 2 (the scores were in base 2).
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const float* __restrict__ part,
                                                             const int32_t* __restrict__ lens, int T, int Hq,
                                                             int Hkv, int G, int S, __nv_bfloat16* __restrict__ o,
                                                             float* __restrict__ lse)
{
    const int bh = blockIdx.x, b = bh / Hq, h = bh % Hq, g = h / G, hh = h % G;
    const int t = threadIdx.x;
    const int len = seq_len(lens, b, T);
    if (len < 1 || len > T) {
        if (t < D) o[(int64_t)bh * D + t] = __float2bfloat16(0.f);
        if (t == 0) lse[bh] = -INFINITY;
        return;
    }
    const float* base = part + ((int64_t)(b * Hkv + g) * S) * G * (D + 2) + hh * (D + 2);
    const int64_t step = (int64_t)G * (D + 2);
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, base[s * step + D]);
    float L = 0.f, acc = 0.f;
    for (int s = 0; s < S; ++s) {
        const float ms = base[s * step + D];
        if (ms == -INFINITY) continue;
        const float w = ex2_approx(ms - M);
        L = fmaf(base[s * step + D + 1], w, L);
        if (t < D) acc = fmaf(base[s * step + t], w, acc);
    }
    if (t < D) o[(int64_t)bh * D + t] = __float2bfloat16(acc / L);
    if (t == 0) lse[bh] = (M + log2f(L)) * kLn2;
}

template <int D, int G>
cudaError_t launch_attn(dim3 grid, const void* q, const void* k, const void* v, const int32_t* lens,
                        const int32_t* idx, const int32_t* nsel, const Problem& pr, float c1, float* part, int S,
                        cudaStream_t st)
{
    const size_t smem = DecSmem<D, G>::kTotal;
    cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    decode_attn_kernel<D, G><<<grid, 128, smem, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                                      (const __nv_bfloat16*)v, lens, idx, nsel, pr.T, pr.Hq,
                                                      pr.Hkv, pr.topk, c1, part, S);
    count_launches(1);
    return cudaSuccess;
}

template <int D>
cudaError_t launch_decode_d(const Problem& pr, const int32_t* lens, const void* q, const void* qp, const void* k,
                            const void* v, const void* kp, int32_t* idx, int32_t* nsel, void* o, float* lse,
                            void* ws, const WsLayout& L, cudaStream_t st)
{
    uint8_t* w = (uint8_t*)ws;
    uint32_t* status = (uint32_t*)(w + L.status);
    float* pooled = (float*)(w + L.pooled);
    float* part = (float*)(w + L.part);
    const int BH = pr.B * pr.Hp;
    {
        dim3 grid((unsigned)((pr.nblk + 7) / 8), (unsigned)BH);
        decode_pool_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)qp, (const __nv_bfloat16*)kp, lens, pr.T,
                                                 pr.Hp, pr.dp, pooled, pr.nblk, status);
        count_launches(1);
    }
    {
        int npad = 1;
        while (npad < pr.nblk || npad < pr.topk) npad <<= 1;
        int tp = 1;
        while (tp < pr.topk) tp <<= 1;
        const size_t smem = (size_t)(npad + tp) * 8;
        cudaError_t e = cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        decode_select_kernel<<<(unsigned)BH, 1024, smem, st>>>(pooled, lens, pr.T, pr.Hp, pr.nblk, npad, pr.topk,
                                                               pr.window, pr.dilation, idx, nsel);
        count_launches(1);
    }
    const int S = decode_splits(pr);
    {
        dim3 grid((unsigned)S, (unsigned)(pr.B * pr.Hkv));
        const float c1 = pr.scale * kLog2eD;
        cudaError_t e = cudaSuccess;
        switch (pr.G) {
        case 1: e = launch_attn<D, 1>(grid, q, k, v, lens, idx, nsel, pr, c1, part, S, st); break;
        case 2: e = launch_attn<D, 2>(grid, q, k, v, lens, idx, nsel, pr, c1, part, S, st); break;
        case 4: e = launch_attn<D, 4>(grid, q, k, v, lens, idx, nsel, pr, c1, part, S, st); break;
        case 8: e = launch_attn<D, 8>(grid, q, k, v, lens, idx, nsel, pr, c1, part, S, st); break;
        default: e = launch_attn<D, 16>(grid, q, k, v, lens, idx, nsel, pr, c1, part, S, st); break;
        }
        if (e != cudaSuccess) return e;
    }
    decode_combine_kernel<D><<<(unsigned)(pr.B * pr.Hq), 128, 0, st>>>(part, lens, pr.T, pr.Hq, pr.Hkv, pr.G, S,
                                                                      (__nv_bfloat16*)o, lse);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

int decode_splits(const Problem& p) { return (p.topk + kSplitBlocks - 1) / kSplitBlocks; }

cudaError_t launch_decode(const Problem& pr, const int32_t* lens, const void* q, const void* qp, const void* k,
                          const void* v, const void* kp, int32_t* idx, int32_t* nsel, void* o, float* lse,
                          void* ws, const WsLayout& L, cudaStream_t st)
{
    if (pr.d == 64) return launch_decode_d<64>(pr, lens, q, qp, k, v, kp, idx, nsel, o, lse, ws, L, st);
    return launch_decode_d<128>(pr, lens, q, qp, k, v, kp, idx, nsel, o, lse, ws, L, st);
}

}  // namespace msa
