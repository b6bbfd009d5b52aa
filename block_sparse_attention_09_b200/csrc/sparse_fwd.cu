// Main Branch forward: exact causal softmax attention (GQA) over the cached
// block selection, producing O and the logsumexp L.
//
// Method (ai-beat post on Flash-MSA training, paragraph 1: the Main Branch
// runs exact softmax over only the selected blocks; "Flash-MSA: Open-Source
// Sparse Attention Kernels Debut", section "How MSA works": GQA main
// attention, block ids cached by the Index Branch).
//
// KV-stationary design over PAIRS of KV blocks.  One CTA owns the blocks 2p
// and 2p+1 of one group: their K and V tiles (2 x 128 keys) are loaded once by
// TMA; the queries that selected either block are gathered from the pair
// index in chunks of 128 rows (128/G tokens x the G query heads of the group,
// head-major: row = hh * 128/G + t) with cp.async into a 2-stage ring.
// Per chunk and block:  S = Q K^T (tcgen05, TMEM) -> P = exp2(S*scale*log2e -
// m_i), zero for a block the row did not select, written back to TMEM as
// bf16 -> O_part += P V (tcgen05 with A from TMEM); then fp32 reductions of
// O_part and of the row sums into global accumulators.  The main cost of a
// KV-stationary forward is on-chip traffic per (row, block) pair -- the query
// gather and the fp32 O reduction -- and a row that selected both blocks of a
// pair pays it once: with selections that favour nearby blocks most rows do.
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

#include <type_traits>

#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kThreads = 512;   // w0 TMA(K,V) | w1 MMA | w2-3 gather | w4-7 softmax of block 2p | w8-11 O out | w12-15 softmax of block 2p+1
constexpr int kGather = 64;     // gather threads
constexpr int kQStages = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kSumLow = 7.703719777548943e-34f;     // 2^-110: row sums outside [kSumLow, kSumHigh]
constexpr float kSumHigh = 1.2676506002282294e30f;    // 2^100   (or not finite) are redone exactly
constexpr float kShiftSlack = 100.f;                  // m_i <= S_ii + kShiftSlack (log2 units)

struct FwdParams {
    int B, T, Hq, Hkv, lgG, tpc, nblk, npair, topk;
    int RB, qb0, per_group;   // query blocks per range; first query block; work items per (b, group)
    float c1;        // scale * log2(e)
    const __nv_bfloat16* q;
    const int32_t* ptr2;
    const int32_t* off2;
    const int32_t* tok2;   // pair lists: (i << 2) | selected 2p | selected 2p+1 << 1
    const float* shift;    // m_i per [b][h][i], log2 units
    float* oacc;
    float* lacc;
    float* bmass;          // nullable: per pair-list entry [e][2][G], the row's weight sum of each block
    uint32_t* status;
};

template <int D>
struct FwdSmem {
    static constexpr uint32_t kTile = 128u * D * 2u;                 // 128 rows x D bf16
    static constexpr uint32_t kKV = 0;                               // K0, V0, K1, V1
    static constexpr uint32_t kQ = 4 * kTile;                        // kQStages query chunks
    static constexpr uint32_t kStg = kQ + kQStages * kTile;          // O staging: half a chunk's tokens
    static constexpr uint32_t kStgBytes = 64u * D * 4u + 1024u;      // 64 rows of D fp32 + 16 B per token
    static constexpr uint32_t kBars = kStg + kStgBytes;
    static constexpr uint32_t kTotal = kBars + 32 * 8 + 16;
    static_assert(kTotal <= 232448, "shared memory per CTA");
};

// One CTA per work item: a pair of KV blocks n0 = 2p, n1 = 2p+1 of one group
// and the queries of one range that selected either.  Chunk c holds 128 rows
// (128/G tokens x the G heads, head-major); per chunk and sub-block s:
//   S_s = Q K_s^T -> TMEM [128 s, 128 s + 128)
//   P_s = exp2(S_s c1 - m_i), zero where the row did not select block n_s or
//         the key is after the query, written back over S_s as bf16
//   O  += P_s V_s (A from TMEM) into one of two O buffers
// so that a row that selected both blocks is gathered once and adds one O
// partial for both.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fwd_main_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, FwdParams p)
{
    using SM = FwdSmem<D>;
    constexpr uint32_t kTile = SM::kTile;
    constexpr int kSlabs = D / 64;
    extern __shared__ __align__(1024) uint8_t smem[];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int qe = 0;
    const RangeItem item = pair_item((int)blockIdx.x, p.nblk, p.npair, p.RB, p.qb0, p.per_group, p.ptr2, p.off2, &qe);
    const int pn = item.n, bg = item.bg;
    const int n0 = 2 * pn, n1 = 2 * pn + 1;
    const int nsub = n1 < qe ? 2 : 1;   // block n1 is read by a query of this range only if n1 < qe
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int G = 1 << p.lgG;
    const int count = item.count;
    if (count <= 0) return;
    const uint32_t code0 = kStTimeoutBase + kKidFwd * 16;
    if ((smem_u32(smem) & 1023u) != 0u) {   // the swizzled tiles need a 1024-byte aligned base
        if (threadIdx.x == 0) atomicCAS(p.status, 0u, code0 + 15);
        return;
    }
    const int32_t* toks = p.tok2 + (int64_t)bg * p.T * p.topk + item.beg;
    const int nchunks = (count + p.tpc - 1) / p.tpc;

    auto k_tile = [&](int s) { return smem + SM::kKV + (uint32_t)(2 * s) * kTile; };
    auto v_tile = [&](int s) { return smem + SM::kKV + (uint32_t)(2 * s + 1) * kTile; };
    uint8_t* q_st = smem + SM::kQ;
    // O staging of half a chunk's tokens: token t' at t' * (G*D*4 + 16) bytes;
    // the 16-byte pad per token spreads the rows of a warp over all banks.
    uint8_t* o_stg = smem + SM::kStg;
    const uint32_t tok_bytes = (uint32_t)G * D * 4u;
    const uint32_t tok_stride = tok_bytes + 16u;
    uint64_t* bars = (uint64_t*)(smem + SM::kBars);
    uint64_t* kv_full = bars;
    uint64_t* q_full = bars + 1;                 // [kQStages]
    uint64_t* q_empty = q_full + kQStages;       // [kQStages]
    uint64_t* s_full = q_empty + kQStages;       // [2] per sub-block
    uint64_t* p_full = s_full + 2;               // [2] per sub-block
    uint64_t* o_full = p_full + 2;               // [2] per O buffer
    uint64_t* o_empty = o_full + 2;              // [2] per O buffer
    uint64_t* fin = o_empty + 2;
    uint32_t* tmem_hold = (uint32_t*)(fin + 1);
    volatile uint32_t* abort_flag = tmem_hold + 1;
    const WaitCtx wc{p.status, abort_flag, MSA_WAIT_LIMIT_NS};

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < kQStages; ++s) { mbar_init(&q_full[s], kGather); mbar_init(&q_empty[s], 1); }
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
    // TMEM columns: S/P of sub-block s at 128 s, O buffers at 256 and 256 + D.

    if (warp == 0) {
        // ---------------- K/V tiles of both blocks (once) ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_arrive_expect_tx(kv_full, 2u * nsub * kTile);
            for (int s = 0; s < nsub; ++s)
                for (int sl = 0; sl < kSlabs; ++sl) {
                    tma_load_4d(k_tile(s) + sl * 16384, &tm_k, kv_full, sl * 64, g, (n0 + s) * 128, b);
                    tma_load_4d(v_tile(s) + sl * 16384, &tm_v, kv_full, sl * 64, g, (n0 + s) * 128, b);
                }
            mbar_drain(kv_full, 0);   // the tiles must have landed before this warp leaves
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
            constexpr uint32_t idPV = idesc_bf16(128, D, false, true);
            const uint32_t qa = smem_u32(q_st);
            // S(c, s) into the columns of sub-block s.  A sub-block's columns
            // still hold P of the previous chunk until its PV MMAs have run, so
            // S(c, s) is issued after PV(c-1, s) (MMAs of one thread run in order).
            auto issue_s = [&](int c, int s) {
                const uint32_t qs = qa + (uint32_t)(c % kQStages) * kTile;
                const uint32_t ka = smem_u32(k_tile(s));
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    umma_ss(tmem + (uint32_t)s * 128u, desc_kmajor(qs, 128, kk * 16), desc_kmajor(ka, 128, kk * 16),
                            idS, kk > 0 ? 1u : 0u);
                umma_commit(&s_full[s]);
                if (s == nsub - 1) umma_commit(&q_empty[c % kQStages]);   // the chunk's queries are read
            };
            auto wait_q = [&](int c) {
                return mbar_wait(&q_full[c % kQStages], (uint32_t)(c / kQStages) & 1u, wc, code0 + 1);
            };
            bool ok = mbar_wait(kv_full, 0, wc, code0 + 0);
            if (ok && nchunks > 0) {
                ok = wait_q(0);
                if (ok) {
                    tc_fence_after();
                    for (int s = 0; s < nsub; ++s) issue_s(0, s);
                }
            }
            for (int c = 0; ok && c < nchunks; ++c) {
                const int buf = c & 1;
                const uint32_t use = (uint32_t)(c >> 1);
                const uint32_t oa = tmem + 256u + (uint32_t)buf * D;
                if (use > 0 && !mbar_wait(&o_empty[buf], (use - 1) & 1u, wc, code0 + 3)) break;
                for (int s = 0; ok && s < nsub; ++s) {
                    if (!mbar_wait(&p_full[s], (uint32_t)c & 1u, wc, code0 + 2)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t pa = tmem + (uint32_t)s * 128u, va = smem_u32(v_tile(s));
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_ts(oa, pa + kk * 8, desc_mnmajor(va, 128, kk * 16), idPV, (s > 0 || kk > 0) ? 1u : 0u);
                    if (s == nsub - 1) umma_commit(&o_full[buf]);
                    if (c + 1 < nchunks) {
                        if (s == 0 && !wait_q(c + 1)) { ok = false; break; }
                        tc_fence_after();
                        issue_s(c + 1, s);
                    }
                }
            }
            umma_commit(fin);
            mbar_drain(fin, 0);
        }
    } else if (warp < 4) {
        // ---------------- query gather (cp.async, 64 threads) ----------------
        const int tid = threadIdx.x - 64;
        constexpr int kPieces = 128 * D / 8;           // 16-byte pieces per chunk
        constexpr int kRowPieces = D / 8;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kQStages;
            const uint32_t use = (uint32_t)(c / kQStages);
            if (use > 0 && !mbar_wait(&q_empty[s], (use - 1) & 1u, wc, code0 + 4)) break;
            const uint32_t qs = smem_u32(q_st + s * kTile);
#pragma unroll 4
            for (int it = 0; it < kPieces / kGather; ++it) {
                const int piece = it * kGather + tid;
                const int row = piece / kRowPieces, ch = piece % kRowPieces;
                const int t = row & (p.tpc - 1), hh = row >> (7 - p.lgG);
                const int jj = c * p.tpc + t;
                const bool valid = jj < count;
                const int i = valid ? (toks[jj] >> 2) : 0;
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
    } else if (warp < 8 || warp >= 12) {
        // ---------------- softmax: P = exp2(S*c1 - m_i) ----------------
        // warps 4-7 take block 2p, warps 12-15 block 2p+1: the two blocks of a
        // chunk are exponentiated at the same time on different warps
        const int r = ((warp & 3) << 5) | lane;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
        const int t = r & (p.tpc - 1), hh = r >> (7 - p.lgG), h = g * G + hh;
        const float* shift_row = p.shift + ((int64_t)b * p.Hq + h) * p.T;
        // this row's entry and shift are loaded one and two chunks ahead, so
        // the dependent global loads overlap the previous chunk's work
        auto ent_of = [&](int cc) { const int jj = cc * p.tpc + t; return jj < count ? toks[jj] : -1; };
        int ent_cur = ent_of(0), ent_nxt = nchunks > 1 ? ent_of(1) : -1;
        float sh_cur = ent_cur >= 0 ? shift_row[ent_cur >> 2] : 0.f;
        for (int c = 0; c < nchunks; ++c) {
            const int ent_nn = c + 2 < nchunks ? ent_of(c + 2) : -1;
            const float sh_nxt = ent_nxt >= 0 ? shift_row[ent_nxt >> 2] : 0.f;
            const bool valid = ent_cur >= 0;
            const int i = valid ? (ent_cur >> 2) : 0;
            const float mh = valid ? sh_cur : 0.f;
            const int flags = valid ? (ent_cur & 3) : 0;
            ent_cur = ent_nxt;
            ent_nxt = ent_nn;
            sh_cur = sh_nxt;
            float l = 0.f;
            bool ok = true;
            const int64_t ent_idx = (int64_t)bg * p.T * p.topk + item.beg + c * p.tpc + t;   // this row's entry
            const int s_first = warp < 8 ? 0 : 1;
            if (s_first >= nsub) break;   // no second block in this item: nothing for this group
            for (int s = s_first; s < s_first + 1; ++s) {
                float ls = 0.f;
                ok = mbar_wait(&s_full[s], (uint32_t)c & 1u, wc, code0 + 5);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                // last key of block n0 + s this row reads (-1: none)
                const int cmax = !((flags >> s) & 1) ? -1 : (((i >> 7) == n0 + s) ? (i & 127) : 127);
                // a block the row did not select gets the shift +inf: every weight
                // becomes exp2(-inf) = 0 with no compare; only a warp holding a
                // diagonal row (keys after the query) takes the masked path
                const float mhs = cmax < 0 ? INFINITY : mh;
                const bool plain = __all_sync(0xffffffffu, cmax < 0 || cmax == 127);
                const uint32_t ta = tmem_addr(tmem, lane_base, (uint32_t)s * 128u);
                // pieces of 32 columns, the next one's load in flight while this one is computed
                uint32_t va[32], vb[32];
                tmem_ld32(ta, va);
#pragma unroll
                for (int piece = 0; piece < 4; ++piece) {
                    uint32_t* v = (piece & 1) ? vb : va;
                    uint32_t pk[16];
                    tmem_ld_wait_regs(v);
                    if (piece + 1 < 4) tmem_ld32(ta + (piece + 1) * 32, (piece & 1) ? va : vb);
                    if (plain) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const float x0 = fmaf(__uint_as_float(v[2 * e]), p.c1, -mhs);
                            const float x1 = fmaf(__uint_as_float(v[2 * e + 1]), p.c1, -mhs);
                            const float p0 = ex2_approx(x0);
                            const float p1 = ex2_approx(x1);
                            pk[e] = pack_bf16x2(p0, p1);
                            // normalise by the weights the PV product actually uses (bf16), so
                            // that O is an exact convex combination of the selected values
                            ls += __uint_as_float(pk[e] << 16) + __uint_as_float(pk[e] & 0xFFFF0000u);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int c0 = piece * 32 + 2 * e;
                            const float p0 = c0 <= cmax ? ex2_approx(fmaf(__uint_as_float(v[2 * e]), p.c1, -mh)) : 0.f;
                            const float p1 =
                                c0 + 1 <= cmax ? ex2_approx(fmaf(__uint_as_float(v[2 * e + 1]), p.c1, -mh)) : 0.f;
                            pk[e] = pack_bf16x2(p0, p1);
                            ls += __uint_as_float(pk[e] << 16) + __uint_as_float(pk[e] & 0xFFFF0000u);
                        }
                    }
                    tmem_st16(ta + piece * 16, pk);   // P overwrites S columns already read
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&p_full[s]);
                l += ls;
                if (p.bmass != nullptr && ((flags >> s) & 1)) p.bmass[(ent_idx * 2 + s) * G + hh] = ls;
            }
            if (!ok) break;
            if (valid) atomicAdd(&p.lacc[((int64_t)b * p.Hq + h) * p.T + i], l);
        }
    } else {
        // ---------------- O partials -> fp32 global accumulators ----------------
        // TMEM -> padded staging in shared memory -> one bulk fp32 reduction of
        // G*D floats per token (whole cache lines at L2 instead of 16-byte
        // reductions from every thread).  The staging holds half a chunk's
        // tokens, so each chunk goes out in two halves.  Rows are head-major,
        // so the eight lanes of one 16-byte store phase hold eight different
        // tokens and the per-token pad puts them on eight different bank groups.
        const int r = ((warp & 3) << 5) | lane;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
        const int t = r & (p.tpc - 1), hh = r >> (7 - p.lgG);
        const int half_tok = p.tpc >> 1;                       // tokens per half
        const int my_half = t >= half_tok ? 1 : 0;
        const int tid = threadIdx.x - 256;                     // token (within a half) this thread reduces
        const uint32_t stg = smem_u32(o_stg);
        const uint32_t my_row = stg + (uint32_t)(t - my_half * half_tok) * tok_stride + (uint32_t)hh * D * 4u;
        auto tok_at = [&](int cc, int hf) {
            const int jj = cc * p.tpc + hf * half_tok + tid;
            return (cc < nchunks && tid < half_tok && jj < count) ? (toks[jj] >> 2) : -1;
        };
        int tk0 = tok_at(0, 0), tk1 = tok_at(0, 1);
        bool issued = false;
        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            const int buf = c & 1;
            const uint32_t use = (uint32_t)(c >> 1);
            ok = mbar_wait(&o_full[buf], use & 1u, wc, code0 + 6);
            const int nt0 = tk0, nt1 = tk1;
            tk0 = tok_at(c + 1, 0);   // next chunk's, loaded early
            tk1 = tok_at(c + 1, 1);
            for (int hf = 0; hf < 2; ++hf) {
                // the previous half's bulk reductions must have read the staging
                if (issued) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                if (!bar_and_sync(2, 128, ok)) { ok = false; break; }   // all four warps go on, or none
                tc_fence_after();
                const uint32_t ta = tmem_addr(tmem, lane_base, 256u + (uint32_t)buf * D);
#pragma unroll
                for (int piece = 0; piece < D / 32; ++piece) {
                    uint32_t v[32];
                    tmem_ld32(ta + piece * 32, v);
                    tmem_ld_wait();
                    if (my_half == hf) {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(my_row + (piece * 32 + 4 * e) * 4),
                                         "r"(v[4 * e]), "r"(v[4 * e + 1]), "r"(v[4 * e + 2]), "r"(v[4 * e + 3])
                                         : "memory");
                    }
                }
                if (hf == 1) {
                    tc_fence_before();
                    mbar_arrive(&o_empty[buf]);     // the TMEM buffer is free once copied out
                }
                fence_proxy_async_smem();
                named_bar_sync(2, 128);
                const int i = hf == 0 ? nt0 : nt1;
                issued = i >= 0;
                if (issued) {
                    float* dst = p.oacc + (((int64_t)b * p.T + i) * p.Hq + g * G) * D;
                    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
                                 "r"(stg + (uint32_t)tid * tok_stride), "r"(tok_bytes)
                                 : "memory");
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                }
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
    // D/32 consecutive elements per lane: one 4- or 8-byte load per row
    using Vec = typename std::conditional<EPL == 4, uint2, uint32_t>::type;
    auto unpack = [](Vec v, float* f) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < EPL / 2; ++e) {
            const float2 x = __bfloat1622float2(h2[e]);
            f[2 * e] = x.x;
            f[2 * e + 1] = x.y;
        }
    };
    float kv[EPL];
    unpack(*reinterpret_cast<const Vec*>(k + (((int64_t)b * T + i) * Hkv + g) * D + lane * EPL), kv);
    const float c1abs = fabsf(c1);
    // the group's G query rows are consecutive: four heads' loads in flight at a time
    const __nv_bfloat16* qg = q + (((int64_t)b * T + i) * Hq + g * G) * D + lane * EPL;
    for (int h0 = 0; h0 < G; h0 += 4) {
        const int nh = min(4, G - h0);
        Vec qv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (u < nh) qv[u] = *reinterpret_cast<const Vec*>(qg + (int64_t)(h0 + u) * D);
        float ss[4], dot[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float x[EPL];
            unpack(u < nh ? qv[u] : Vec{}, x);
            ss[u] = 0.f;
            dot[u] = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                ss[u] = fmaf(x[e], x[e], ss[u]);
                dot[u] = fmaf(x[e], kv[e], dot[u]);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
                dot[u] += __shfl_xor_sync(0xffffffffu, dot[u], off);
            }
        }
        if (lane < nh) {
            float su = ss[0], du = dot[0];
#pragma unroll
            for (int u = 1; u < 4; ++u)
                if (lane == u) { su = ss[u]; du = dot[u]; }
            const int h = g * G + h0 + lane;
            shift[((int64_t)b * Hq + h) * T + i] = fminf(c1abs * sqrtf(su) * km, c1 * du + kShiftSlack);
        }
    }
}

// O = O_acc / l (bf16), L = (m + log2 l) ln 2 for the computed rows (q0 ..
// T-1); rows whose l is outside [kSumLow, kSumHigh] or not finite are listed
// (count in status word 2).
template <int D, bool Small>
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
    int b, i, h;
    active_coords<Small>(ar, T, Hq, q0, b, i, h);
    const int64_t row = ((int64_t)b * T + i) * Hq + h;
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
                         float* bmass, cudaStream_t st)
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
    p.tpc = 128 / pr.G; p.nblk = pr.nblk; p.npair = pair_count(pr.nblk); p.topk = pr.topk;
    p.c1 = c1;
    p.q = qb;
    p.ptr2 = (const int32_t*)(w + L.ptr2);
    p.off2 = (const int32_t*)(w + L.cnt2);
    p.tok2 = (const int32_t*)(w + L.tok2);
    p.shift = shift; p.oacc = oacc; p.lacc = lacc; p.bmass = bmass;
    p.status = (uint32_t*)(w + L.status);
    p.RB = range_blocks(pr);
    p.qb0 = pr.qb0;
    p.per_group = pair_items_per_group(pr.nblk, p.RB, pr.qb0);
    const size_t smem = FwdSmem<D>::kTotal;
    if ((e = cudaFuncSetAttribute(fwd_main_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess)
        return e;
    trace_begin(kTraceFwdMain, st);
    fwd_main_kernel<D><<<(unsigned)(p.per_group * pr.B * pr.Hkv), kThreads, smem, st>>>(tm_k, tm_v, p);
    count_launches(1);
    trace_end(kTraceFwdMain, st);

    const int64_t fth = pr.rows_q_active() * (D / 8);
    if (fth < ((int64_t)1 << 31))
        fwd_finalize_kernel<D, true><<<(unsigned)((fth + 255) / 256), 256, 0, st>>>(
            oacc, lacc, shift, pr.B, pr.T, pr.Hq, pr.q0, (__nv_bfloat16*)o, lse, nflag, flags);
    else
        fwd_finalize_kernel<D, false><<<(unsigned)((fth + 255) / 256), 256, 0, st>>>(
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
                       float* bmass, cudaStream_t st)
{
    if (pr.d == 64) return launch_fwd_d<64>(pr, q, k, v, tm_k, tm_v, idx, nsel, o, lse, ws, L, bmass, st);
    return launch_fwd_d<128>(pr, q, k, v, tm_k, tm_v, idx, nsel, o, lse, ws, L, bmass, st);
}

}  // namespace msa
