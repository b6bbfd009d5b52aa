// Main Branch forward: exact causal softmax attention (GQA) over the cached
// block selection, producing O and the logsumexp L.
//
// Method (ai-beat post on Flash-MSA training, paragraph 1: the Main Branch
// runs exact softmax over only the selected blocks; "Flash-MSA: Open-Source
// Sparse Attention Kernels Debut", section "How MSA works": GQA main
// attention, block ids cached by the Index Branch).
//
// KV-stationary design.  One CTA owns one KV block n of one group: its K and
// V tiles (128 keys) are loaded once by TMA; the queries that selected the
// block are gathered from the inverse index in chunks of 128 rows (128/G
// tokens x the G query heads of the group, head-major: row = hh * 128/G + t)
// with cp.async into a 3-stage ring.
// Per chunk:  S = Q K^T (tcgen05, TMEM) -> P = exp2(S*scale*log2e - m_i) written
// back to TMEM as bf16 -> O_part = P V (tcgen05 with A from TMEM) -> fp32
// reductions of O_part and of the row sums into global accumulators.
//
// Softmax normalisation across the CTAs that share a query row uses a fixed
// per-row shift m_i instead of a running maximum, so every CTA's partial sums
// are directly additive.  m_i only has to lie near the row's true maximum
// score (in log2 units, within what fp32 exponents absorb), and it is
// bracketed by two values known before any CTA starts:
//   U_i = |scale| |q_i| max over the row's selected blocks of max |k_j|
//         (Cauchy-Schwarz: no score of the row is above it), and
//   S_ii = the score of the query's own key, which every row reads (own
//         block forced, j = i visible): the row maximum is at least S_ii.
// With m_i = min(U_i, S_ii + 100) (log2 units) the largest weight
// exp2(S - m_i) is in [2^-100, 1] unless the row's best score exceeds S_ii
// by more than 100 (then m_i = S_ii + 100 and weights may grow large).  A
// single large-norm key therefore no longer loosens the shift of the rows
// that read it.  The finalize pass divides by the row sum and sets
// L = (m_i + log2 sum) ln 2.  Rows whose sum is outside [2^-110, 2^100] (or
// not finite) are listed and recomputed exactly by a fallback kernel with a
// two-pass softmax.
#include <math.h>

#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kThreads = 448;   // w0 TMA(K,V) | w1 MMA | w2-5 gather | w6-9 softmax | w10-13 O out
constexpr int kQStages = 3;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kSumLow = 7.703719777548943e-34f;     // 2^-110: row sums outside [kSumLow, kSumHigh]
constexpr float kSumHigh = 1.2676506002282294e30f;    // 2^100   (or not finite) are redone exactly
constexpr float kShiftSlack = 100.f;                  // m_i <= S_ii + kShiftSlack (log2 units)

struct FwdParams {
    int B, T, Hq, Hkv, lgG, tpc, nblk, topk;
    int RB, qb0, per_group;   // query blocks per range; first query block; work items per (b, group)
    float c1;        // scale * log2(e)
    const __nv_bfloat16* q;
    const int32_t* ptr;
    const int32_t* off;
    const int32_t* tok;
    const float* shift;   // m_i per [b][h][i], log2 units
    float* oacc;
    float* lacc;
    uint32_t* status;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fwd_main_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                FwdParams p)
{
    constexpr uint32_t kTile = 128u * D * 2u;   // 128 rows x D bf16
    constexpr int kSlabs = D / 64;
    extern __shared__ __align__(1024) uint8_t smem[];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const RangeItem item = range_item((int)blockIdx.x, p.nblk, p.RB, p.qb0, p.per_group, p.ptr, p.off);
    const int n = item.n, bg = item.bg;
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int G = 1 << p.lgG;
    const int count = item.count;
    if (count <= 0) return;
    const uint32_t code0 = kStTimeoutBase + kKidFwd * 16;
    if ((smem_u32(smem) & 1023u) != 0u) {   // the swizzled tiles need a 1024-byte aligned base
        if (threadIdx.x == 0) atomicCAS(p.status, 0u, code0 + 15);
        return;
    }
    const int32_t* toks = p.tok + (int64_t)bg * p.T * p.topk + item.beg;
    const int nchunks = (count + p.tpc - 1) / p.tpc;

    uint8_t* k_tile = smem;
    uint8_t* v_tile = smem + kTile;
    uint8_t* q_st = smem + 2 * kTile;
    // O staging: token t of a chunk at t * (G*D*4 + 16) bytes; the 16-byte pad
    // per token spreads the rows of a warp over all banks.
    uint8_t* o_stg = q_st + kQStages * kTile;
    const uint32_t tok_bytes = (uint32_t)G * D * 4u;
    const uint32_t tok_stride = tok_bytes + 16u;
    uint64_t* bars = (uint64_t*)(o_stg + 128 * D * 4 + 2048);
    uint64_t* kv_full = bars;
    uint64_t* q_full = bars + 1;
    uint64_t* q_empty = q_full + kQStages;
    uint64_t* s_full = q_empty + kQStages;
    uint64_t* p_full = s_full + 2;
    uint64_t* o_full = p_full + 2;
    uint64_t* o_empty = o_full + 2;
    uint64_t* fin = o_empty + 2;
    uint32_t* tmem_hold = (uint32_t*)(fin + 1);
    volatile uint32_t* abort_flag = tmem_hold + 1;
    const WaitCtx wc{p.status, abort_flag, MSA_WAIT_LIMIT_NS};

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < kQStages; ++s) { mbar_init(&q_full[s], 128); mbar_init(&q_empty[s], 1); }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 128);
            mbar_init(&o_full[s], 1);
            mbar_init(&o_empty[s], 128);
        }
        mbar_init(fin, 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 1) { tmem_alloc(tmem_hold, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_hold;
    // TMEM columns: S/P buffers at 0 and 128, O buffers at 256 and 256 + D.

    if (warp == 0) {
        // ---------------- K/V tiles (once) ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_arrive_expect_tx(kv_full, 2 * kTile);
            for (int s = 0; s < kSlabs; ++s) {
                tma_load_4d(k_tile + s * 16384, &tm_k, kv_full, s * 64, g, n * 128, b);
                tma_load_4d(v_tile + s * 16384, &tm_v, kv_full, s * 64, g, n * 128, b);
            }
            mbar_drain(kv_full, 0);   // the tiles must have landed before this warp leaves
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idPV = idesc_bf16(128, D, false, true);
            const uint32_t ka = smem_u32(k_tile), va = smem_u32(v_tile), qa = smem_u32(q_st);
            // S(c+2) reuses the TMEM columns where P(c) lives, so it is issued
            // only after every K-step of PV(c) (MMAs of one thread run in order).
            auto issue_s = [&](int c) -> bool {
                const int s = c % kQStages;
                const uint32_t use = (uint32_t)(c / kQStages);
                if (!mbar_wait(&q_full[s], use & 1u, wc, code0 + 1)) return false;
                tc_fence_after();
                const uint32_t qs = qa + s * kTile;
                const uint32_t dS = tmem + (uint32_t)(c & 1) * 128u;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    umma_ss(dS, desc_kmajor(qs, 128, kk * 16), desc_kmajor(ka, 128, kk * 16), idS,
                            kk > 0 ? 1u : 0u);
                umma_commit(&q_empty[s]);
                umma_commit(&s_full[c & 1]);
                return true;
            };
            bool ok = mbar_wait(kv_full, 0, wc, code0 + 0);
            if (ok && nchunks > 0) ok = issue_s(0);
            if (ok && nchunks > 1) ok = issue_s(1);
            for (int c = 0; ok && c < nchunks; ++c) {
                const int buf = c & 1;
                const uint32_t use = (uint32_t)(c >> 1);
                if (!mbar_wait(&p_full[buf], use & 1u, wc, code0 + 2)) break;
                if (use > 0 && !mbar_wait(&o_empty[buf], (use - 1) & 1u, wc, code0 + 3)) break;
                tc_fence_after();
                const uint32_t pa = tmem + (uint32_t)buf * 128u;
                const uint32_t oa = tmem + 256u + (uint32_t)buf * D;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(oa, pa + kk * 8, desc_mnmajor(va, 128, kk * 16), idPV, kk > 0 ? 1u : 0u);
                umma_commit(&o_full[buf]);
                if (c + 2 < nchunks) ok = issue_s(c + 2);
            }
            umma_commit(fin);
            mbar_drain(fin, 0);
        }
    } else if (warp < 6) {
        // ---------------- query gather (cp.async, 128 threads) ----------------
        const int tid = threadIdx.x - 64;
        constexpr int kPieces = 128 * D / 8;           // 16-byte pieces per chunk
        constexpr int kRowPieces = D / 8;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kQStages;
            const uint32_t use = (uint32_t)(c / kQStages);
            if (use > 0 && !mbar_wait(&q_empty[s], (use - 1) & 1u, wc, code0 + 4)) break;
            const uint32_t qs = smem_u32(q_st + s * kTile);
#pragma unroll 4
            for (int it = 0; it < kPieces / 128; ++it) {
                const int piece = it * 128 + tid;
                const int row = piece / kRowPieces, ch = piece % kRowPieces;
                const int t = row & (p.tpc - 1), hh = row >> (7 - p.lgG);
                const int jj = c * p.tpc + t;
                const bool valid = jj < count;
                const int i = valid ? toks[jj] : 0;
                const __nv_bfloat16* src =
                    p.q + (((int64_t)b * p.T + i) * p.Hq + g * G + hh) * D + ch * 8;
                cp_async_16(qs + sw128_offset(row, ch & 7, ch >> 3, 128), src, valid ? 16u : 0u);
            }
            cp_async_commit();
            cp_async_wait<0>();
            fence_proxy_async_smem();
            mbar_arrive(&q_full[s]);
        }
        cp_async_wait<0>();
    } else if (warp < 10) {
        // ---------------- softmax: P = exp2(S*c1 - m_i) ----------------
        const int r = ((warp & 3) << 5) | lane;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
        const int t = r & (p.tpc - 1), hh = r >> (7 - p.lgG), h = g * G + hh;
        const float* shift_row = p.shift + ((int64_t)b * p.Hq + h) * p.T;
        // this row's token and shift are loaded one and two chunks ahead, so
        // the dependent global loads overlap the previous chunk's work
        auto tok_of = [&](int cc) { const int jj = cc * p.tpc + t; return jj < count ? toks[jj] : -1; };
        int tok_cur = tok_of(0), tok_nxt = nchunks > 1 ? tok_of(1) : -1;
        float sh_cur = tok_cur >= 0 ? shift_row[tok_cur] : 0.f;
        for (int c = 0; c < nchunks; ++c) {
            const int buf = c & 1;
            const uint32_t use = (uint32_t)(c >> 1);
            const int tok_nn = c + 2 < nchunks ? tok_of(c + 2) : -1;
            const float sh_nxt = tok_nxt >= 0 ? shift_row[tok_nxt] : 0.f;
            const bool ok = mbar_wait(&s_full[buf], use & 1u, wc, code0 + 5);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const bool valid = tok_cur >= 0;
            const int i = valid ? tok_cur : 0;
            const int cmax = valid ? (((i >> 7) == n) ? (i & 127) : 127) : -1;
            const float mh = valid ? sh_cur : 0.f;
            tok_cur = tok_nxt;
            tok_nxt = tok_nn;
            sh_cur = sh_nxt;
            const uint32_t ta = tmem_addr(tmem, lane_base, (uint32_t)buf * 128u);
            float l = 0.f;
#pragma unroll
            for (int piece = 0; piece < 4; ++piece) {
                uint32_t v[32], pk[16];
                tmem_ld32(ta + piece * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int c0 = piece * 32 + 2 * e;
                    const float p0 = c0 <= cmax ? ex2_approx(fmaf(__uint_as_float(v[2 * e]), p.c1, -mh)) : 0.f;
                    const float p1 = c0 + 1 <= cmax ? ex2_approx(fmaf(__uint_as_float(v[2 * e + 1]), p.c1, -mh)) : 0.f;
                    pk[e] = pack_bf16x2(p0, p1);
                    // normalise by the weights the PV product actually uses (bf16), so
                    // that O is an exact convex combination of the selected values
                    l += __uint_as_float(pk[e] << 16) + __uint_as_float(pk[e] & 0xFFFF0000u);
                }
                tmem_st16(ta + piece * 16, pk);   // P overwrites S columns already read
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&p_full[buf]);
            if (valid) atomicAdd(&p.lacc[((int64_t)b * p.Hq + h) * p.T + i], l);
        }
    } else {
        // ---------------- O partials -> fp32 global accumulators ----------------
        // TMEM -> padded staging in shared memory -> one bulk fp32 reduction of
        // G*D floats per token (whole cache lines at L2 instead of 16-byte
        // reductions from every thread).  Rows are head-major, so the eight
        // lanes of one 16-byte store phase hold eight different tokens and the
        // per-token pad puts them on eight different bank groups.
        const int r = ((warp & 3) << 5) | lane;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
        const int t = r & (p.tpc - 1), hh = r >> (7 - p.lgG);
        const int tid = threadIdx.x - 320;             // token this thread reduces
        const uint32_t stg = smem_u32(o_stg);
        const uint32_t my_row = stg + (uint32_t)t * tok_stride + (uint32_t)hh * D * 4u;
        int my_tok_id = tid < min(p.tpc, count) ? toks[tid] : 0;
        bool issued = false;
        for (int c = 0; c < nchunks; ++c) {
            const int buf = c & 1;
            const uint32_t use = (uint32_t)(c >> 1);
            const bool ok = mbar_wait(&o_full[buf], use & 1u, wc, code0 + 6);
            // the previous chunk's bulk reductions must have read the staging
            if (issued) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            if (!bar_and_sync(2, 128, ok)) break;   // all four warps go on, or none
            tc_fence_after();
            const uint32_t ta = tmem_addr(tmem, lane_base, 256u + (uint32_t)buf * D);
#pragma unroll
            for (int piece = 0; piece < D / 32; ++piece) {
                uint32_t v[32];
                tmem_ld32(ta + piece * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(my_row + (piece * 32 + 4 * e) * 4),
                                 "r"(v[4 * e]), "r"(v[4 * e + 1]), "r"(v[4 * e + 2]), "r"(v[4 * e + 3])
                                 : "memory");
            }
            tc_fence_before();
            mbar_arrive(&o_empty[buf]);     // the TMEM buffer is free once copied out
            fence_proxy_async_smem();
            named_bar_sync(2, 128);
            const int ntok = min(p.tpc, count - c * p.tpc);
            const int i = my_tok_id;
            my_tok_id = (c + 1 < nchunks && tid < p.tpc && (c + 1) * p.tpc + tid < count)
                            ? toks[(c + 1) * p.tpc + tid] : 0;   // next chunk's, loaded early
            issued = tid < ntok;
            if (issued) {
                float* dst = p.oacc + (((int64_t)b * p.T + i) * p.Hq + g * G) * D;
                asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
                             "r"(stg + (uint32_t)tid * tok_stride), "r"(tok_bytes)
                             : "memory");
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
        }
        // the staging must have been read before the CTA exits; the global
        // side completes on its own
        if (issued) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// max |k_j| per KV block: grid (nblk, B*Hkv), one CTA per block of 128 keys
// (keys past T are not read); D/8 lanes per key row.
template <int D>
__global__ void __launch_bounds__(256) fwd_kmax_kernel(const __nv_bfloat16* __restrict__ k, int T, int Hkv,
                                                       int nblk, float* __restrict__ kmax_blk)
{
    constexpr int LPR = D / 8, RPP = 256 / LPR;   // lanes per row, rows per pass
    __shared__ float red[8];
    const int n = blockIdx.x, bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;
    const int sub = threadIdx.x % LPR, r = threadIdx.x / LPR;
    float mx = 0.f;
    // the same number of passes for every lane: the shuffles below need the
    // whole warp, and rows past T are predicated off instead
    for (int pass = 0; pass < 128 / RPP; ++pass) {
        const int t = n * 128 + pass * RPP + r;
        float ss = 0.f;
        if (t < T) {
            const uint4 u = *reinterpret_cast<const uint4*>(k + (((int64_t)b * T + t) * Hkv + g) * D + sub * 8);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                ss = fmaf(f.x, f.x, ss);
                ss = fmaf(f.y, f.y, ss);
            }
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        mx = fmaxf(mx, ss);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = red[0];
        for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
        kmax_blk[(int64_t)bg * nblk + n] = sqrtf(m);
    }
}

// Per-row softmax shift m_i (log2 units) for the computed rows q0 .. T-1:
// one warp per (b, group, query i) serves the G heads of the group, which
// share the selection.  U = |c1| |q| max over the selected blocks of their
// max |k|; S_ii = c1 q_i . k_i (the own key); m = min(U, S_ii + slack).
// Selection entries outside [0, i/128] are skipped here (the inverse index
// reports them).
template <int D>
__global__ void __launch_bounds__(256) fwd_shift_kernel(const __nv_bfloat16* __restrict__ q,
                                                        const __nv_bfloat16* __restrict__ k,
                                                        const int32_t* __restrict__ idx,
                                                        const int32_t* __restrict__ nsel,
                                                        const float* __restrict__ kmax_blk, int B, int T, int Hq,
                                                        int Hkv, int topk, int nblk, int q0, float c1,
                                                        float* __restrict__ shift)
{
    constexpr int EPL = D / 32;   // elements per lane
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int Tq = T - q0;
    if (w >= (int64_t)B * Hkv * Tq) return;   // warp-uniform
    const int bg = (int)(w / Tq), i = q0 + (int)(w % Tq);
    const int b = bg / Hkv, g = bg % Hkv, G = Hq / Hkv;
    const int64_t srow = (int64_t)bg * T + i;
    int ns = nsel[srow];
    ns = ns < 0 ? 0 : (ns > topk ? topk : ns);
    float km = 0.f;
    for (int s = lane; s < ns; s += 32) {
        const int n = idx[srow * topk + s];
        if (n >= 0 && n <= (i >> 7)) km = fmaxf(km, kmax_blk[(int64_t)bg * nblk + n]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) km = fmaxf(km, __shfl_xor_sync(0xffffffffu, km, off));
    float kv[EPL];
    {
        const __nv_bfloat16* kr = k + (((int64_t)b * T + i) * Hkv + g) * D + lane * EPL;
#pragma unroll
        for (int e = 0; e < EPL; ++e) kv[e] = __bfloat162float(kr[e]);
    }
    const float c1abs = fabsf(c1);
    for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        const __nv_bfloat16* qr = q + (((int64_t)b * T + i) * Hq + h) * D + lane * EPL;
        float ss = 0.f, dot = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            const float x = __bfloat162float(qr[e]);
            ss = fmaf(x, x, ss);
            dot = fmaf(x, kv[e], dot);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, off);
            dot += __shfl_xor_sync(0xffffffffu, dot, off);
        }
        if (lane == 0)
            shift[((int64_t)b * Hq + h) * T + i] = fminf(c1abs * sqrtf(ss) * km, c1 * dot + kShiftSlack);
    }
}

// O = O_acc / l (bf16), L = (m + log2 l) ln 2 for the computed rows (q0 ..
// T-1); rows whose l is outside [kSumLow, kSumHigh] or not finite are listed
// (count in status word 2).
template <int D>
__global__ void __launch_bounds__(256) fwd_finalize_kernel(const float* __restrict__ oacc,
                                                           const float* __restrict__ lacc,
                                                           const float* __restrict__ shift, int B, int T,
                                                           int Hq, int q0, __nv_bfloat16* __restrict__ o,
                                                           float* __restrict__ lse, uint32_t* nflag, int* flags)
{
    constexpr int LPR = D / 8;
    constexpr float kLn2 = 0.6931471805599453f;
    const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t ar = gt / LPR;
    const int sub = (int)(gt % LPR);
    if (ar >= (int64_t)B * (T - q0) * Hq) return;
    const int64_t row = active_row(ar, T, Hq, q0);   // (b*T + i)*Hq + h
    const int h = (int)(row % Hq);
    const int64_t bi = row / Hq;
    const int i = (int)(bi % T), b = (int)(bi / T);
    const int64_t lrow = ((int64_t)b * Hq + h) * T + i;
    const float l = lacc[lrow];
    const float inv = 1.f / l;
    const float4 a = *reinterpret_cast<const float4*>(oacc + row * D + sub * 8);
    const float4 c = *reinterpret_cast<const float4*>(oacc + row * D + sub * 8 + 4);
    uint4 out;
    out.x = pack_bf16x2(a.x * inv, a.y * inv);
    out.y = pack_bf16x2(a.z * inv, a.w * inv);
    out.z = pack_bf16x2(c.x * inv, c.y * inv);
    out.w = pack_bf16x2(c.z * inv, c.w * inv);
    *reinterpret_cast<uint4*>(o + row * D + sub * 8) = out;
    if (sub == 0) {
        lse[lrow] = (shift[lrow] + log2f(l)) * kLn2;
        if (!(l >= kSumLow && l <= kSumHigh)) flags[atomicAdd(nflag, 1u)] = (int)row;
    }
}

// Exact two-pass softmax for the listed rows (rare: a row whose best score is
// more than the shift slack above its own key's score).  One warp per row.
template <int D>
__global__ void __launch_bounds__(128) fwd_fallback_kernel(const __nv_bfloat16* __restrict__ q,
                                                           const __nv_bfloat16* __restrict__ k,
                                                           const __nv_bfloat16* __restrict__ v,
                                                           const int32_t* __restrict__ idx,
                                                           const int32_t* __restrict__ nsel, int B, int T,
                                                           int Hq, int Hkv, int topk, float scale,
                                                           const uint32_t* nflag, const int* flags,
                                                           __nv_bfloat16* __restrict__ o,
                                                           float* __restrict__ lse)
{
    __shared__ float qs[4][D];
    __shared__ float ps[4][32];
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = Hq / Hkv;
    const int nf = (int)*nflag;
    for (int f = blockIdx.x * 4 + w; f < nf; f += gridDim.x * 4) {
        const int64_t row = flags[f];
        const int h = (int)(row % Hq);
        const int64_t bi = row / Hq;
        const int i = (int)(bi % T), b = (int)(bi / T);
        const int g = h / G, bg = b * Hkv + g;
        for (int e = lane; e < D; e += 32) qs[w][e] = __bfloat162float(q[row * D + e]);
        __syncwarp();
        const int64_t srow = (int64_t)bg * T + i;
        int ns = nsel[srow];
        ns = ns < 0 ? 0 : (ns > topk ? topk : ns);
        const int32_t* sel = idx + srow * topk;
        auto score = [&](int j) {
            const __nv_bfloat16* kr = k + (((int64_t)b * T + j) * Hkv + g) * D;
            float acc = 0.f;
            for (int e = 0; e < D; ++e) acc = fmaf(qs[w][e], __bfloat162float(kr[e]), acc);
            return acc * scale;
        };
        float m = -INFINITY;
        int prev = -1;
        for (int s = 0; s < ns; ++s) {
            const int nb = sel[s];
            if (nb < 0 || nb > (i >> 7) || nb <= prev) continue;
            prev = nb;
            const int jend = min(nb * 128 + 128, i + 1);
            for (int j = nb * 128 + lane; j < jend; j += 32) m = fmaxf(m, score(j));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float l = 0.f, acc[D / 32];
#pragma unroll
        for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;
        prev = -1;
        for (int s = 0; s < ns; ++s) {
            const int nb = sel[s];
            if (nb < 0 || nb > (i >> 7) || nb <= prev) continue;
            prev = nb;
            const int jend = min(nb * 128 + 128, i + 1);
            for (int jb = nb * 128; jb < jend; jb += 32) {
                const int j = jb + lane;
                const float pe = j < jend ? expf(score(j) - m) : 0.f;
                l += pe;
                ps[w][lane] = pe;
                __syncwarp();
                const int cnt = min(32, jend - jb);
                for (int kk = 0; kk < cnt; ++kk) {
                    const __nv_bfloat16* vr = v + (((int64_t)b * T + jb + kk) * Hkv + g) * D;
#pragma unroll
                    for (int e = 0; e < D / 32; ++e)
                        acc[e] = fmaf(ps[w][kk], __bfloat162float(vr[lane + 32 * e]), acc[e]);
                }
                __syncwarp();
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
        for (int e = 0; e < D / 32; ++e) o[row * D + lane + 32 * e] = __float2bfloat16(acc[e] / l);
        if (lane == 0) lse[((int64_t)b * Hq + h) * T + i] = m + logf(l);
        __syncwarp();
    }
}

template <int D>
cudaError_t launch_fwd_d(const Problem& pr, const void* q, const void* k, const void* v,
                         const CUtensorMap& tm_k, const CUtensorMap& tm_v, const int32_t* idx,
                         const int32_t* nsel, void* o, float* lse, void* ws, const WsLayout& L,
                         cudaStream_t st)
{
    uint8_t* w = (uint8_t*)ws;
    float* shift = (float*)(w + L.shift);
    float* kmax = (float*)(w + L.kmax);
    float* oacc = (float*)(w + L.oacc);
    float* lacc = (float*)(w + L.lacc);
    uint32_t* nflag = (uint32_t*)(w + L.status) + 2;   // cleared with the status words by the caller
    int* flags = (int*)(w + L.flags);
    const __nv_bfloat16* qb = (const __nv_bfloat16*)q;
    const __nv_bfloat16* kb = (const __nv_bfloat16*)k;
    const float c1 = pr.scale * kLog2e;
    cudaError_t e;
    if ((e = cudaMemsetAsync(oacc, 0, sizeof(float) * (size_t)pr.rows_q() * D, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(lacc, 0, sizeof(float) * (size_t)pr.rows_q(), st)) != cudaSuccess) return e;

    fwd_kmax_kernel<D><<<dim3((unsigned)pr.nblk, (unsigned)(pr.B * pr.Hkv)), 256, 0, st>>>(kb, pr.T, pr.Hkv,
                                                                                      pr.nblk, kmax);
    count_launches(1);
    const int64_t warps = (int64_t)pr.B * pr.Hkv * (pr.T - pr.q0);
    fwd_shift_kernel<D><<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(qb, kb, idx, nsel, kmax, pr.B, pr.T, pr.Hq,
                                                                    pr.Hkv, pr.topk, pr.nblk, pr.q0, c1, shift);
    count_launches(1);

    FwdParams p;
    p.B = pr.B; p.T = pr.T; p.Hq = pr.Hq; p.Hkv = pr.Hkv;
    p.lgG = 31 - __builtin_clz((unsigned)pr.G);
    p.tpc = 128 / pr.G; p.nblk = pr.nblk; p.topk = pr.topk;
    p.c1 = c1;
    p.q = qb;
    p.ptr = (const int32_t*)(w + L.ptr);
    p.off = (const int32_t*)(w + L.cnt);
    p.tok = (const int32_t*)(w + L.tok);
    p.shift = shift; p.oacc = oacc; p.lacc = lacc;
    p.status = (uint32_t*)(w + L.status);
    p.RB = range_blocks(pr);
    p.qb0 = pr.qb0;
    p.per_group = range_items_per_group(pr.nblk, p.RB, pr.qb0);
    const size_t smem = (size_t)(2 + kQStages) * 128 * D * 2 + 128 * D * 4 + 2048 + 32 * 8;
    if ((e = cudaFuncSetAttribute(fwd_main_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess)
        return e;
    trace_begin(kTraceFwdMain, st);
    fwd_main_kernel<D><<<(unsigned)(p.per_group * pr.B * pr.Hkv), kThreads, smem, st>>>(tm_k, tm_v, p);
    count_launches(1);
    trace_end(kTraceFwdMain, st);

    const int64_t fth = pr.rows_q_active() * (D / 8);
    fwd_finalize_kernel<D><<<(unsigned)((fth + 255) / 256), 256, 0, st>>>(
        oacc, lacc, shift, pr.B, pr.T, pr.Hq, pr.q0, (__nv_bfloat16*)o, lse, nflag, flags);
    count_launches(1);
    fwd_fallback_kernel<D><<<148, 128, 0, st>>>(qb, kb, (const __nv_bfloat16*)v, idx, nsel, pr.B,
                                                pr.T, pr.Hq, pr.Hkv, pr.topk, pr.scale, nflag, flags,
                                                (__nv_bfloat16*)o, lse);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd(const Problem& pr, const void* q, const void* k, const void* v,
                       const CUtensorMap& tm_k, const CUtensorMap& tm_v, const int32_t* idx,
                       const int32_t* nsel, void* o, float* lse, void* ws, const WsLayout& L,
                       cudaStream_t st)
{
    if (pr.d == 64) return launch_fwd_d<64>(pr, q, k, v, tm_k, tm_v, idx, nsel, o, lse, ws, L, st);
    return launch_fwd_d<128>(pr, q, k, v, tm_k, tm_v, idx, nsel, o, lse, ws, L, st);
}

}  // namespace msa
