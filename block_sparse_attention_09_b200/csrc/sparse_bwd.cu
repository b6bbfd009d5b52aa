// Main Branch backward: dQ, dK, dV of the block-sparse causal GQA attention
// from dO, reusing the cached block selection and the forward's logsumexp.
//
// Method (ai-beat post on Flash-MSA training, paragraph 2: training through
// the sparse pattern needs custom backward kernels; the selection itself is
// piecewise constant, so no gradient reaches the proxy inputs).
//
// With P = exp(S - L), D_i = dO_i . O_i, dS = P (dO V^T - D) * scale:
//   dV = P^T dO,  dK = dS^T Q,  dQ = dS K.
//
// KV-stationary: one CTA owns KV block n of one group, keeps K and V in
// shared memory and dK, dV as fp32 accumulators in TMEM for the whole
// bucket, so dK/dV need no atomics.  Chunks of 128 query rows (128/G tokens
// x G heads) are gathered with cp.async (Q, dO, plus each row's L, D and
// causal limit) into a 2-stage ring.  Per chunk, in the transposed
// orientation so that one TMEM lane is one key:
//   S^T = K Q^T, dP^T = V dO^T                 (tcgen05, A and B in smem)
//   P^T, dS^T  -> TMEM (bf16) and dS^T -> smem  (softmax warps, lane = key)
//   dV += P^T dO, dK += dS^T Q                  (tcgen05, A from TMEM)
//   dQ_part = dS K                              (tcgen05, A = dS from smem)
//   dQ_part -> fp32 reductions into a global accumulator (lane = query row).
#include <math.h>

#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kThreads = 448;   // w0 TMA(K,V) | w1 MMA | w2-5 gather | w6-9 dS | w10-13 dQ, dK/dV out
constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
    int B, T, Hq, Hkv, lgG, tpc, nblk, topk;
    int RB, per_group;   // query blocks per range; work items per (b, group)
    float c1;      // scale * log2(e)
    float scale;
    const __nv_bfloat16* q;
    const __nv_bfloat16* dout;
    const float* lse;
    const float* dsum;
    const int32_t* ptr;
    const int32_t* off;
    const int32_t* tok;
    float* dqacc;
    float* dkacc;    // fp32 dK, dV accumulators [B][T][Hkv][D]: one partial per item
    float* dvacc;
    uint32_t* status;
};

template <int D>
struct BwdSmem {
    static constexpr int kStages = 4;                           // Q/dO ring
    static constexpr uint32_t kKV = 128u * D * 2u;              // one K or V tile
    static constexpr uint32_t kHalf = 64u * D * 2u;             // Q or dO of one 64-row chunk
    static constexpr uint32_t kK = 0, kV = kKV;
    static constexpr uint32_t kStage0 = 2 * kKV;                // stage s: Q at s*2*kHalf, dO after it
    static constexpr uint32_t kDS = kStage0 + kStages * 2 * kHalf;   // 2 dS tiles (128 keys x 64 rows)
    static constexpr uint32_t kDSTile = 128u * 64u * 2u;
    static constexpr uint32_t kMeta = kDS + 2 * kDSTile;        // per stage {L2[64], D[64], cmax[64]}
    static constexpr uint32_t kMetaStage = 64 * 4 * 2 + 64;
    static constexpr uint32_t kBars = kMeta + kStages * kMetaStage;
    static constexpr uint32_t kNumBars = 1 + 2 * kStages + 5 * 2 + 2;
    static constexpr uint32_t kTotal = kBars + kNumBars * 8 + 8;
    static_assert(2 * 128 * (D * 4 + 16) <= kMeta - kStage0, "dK/dV staging must fit the stage and dS area");
};

// Work per item: the 64-row chunks (64/G tokens x G heads) of the item's
// queries, software-pipelined over two TMEM buffer sets:
//   MMA:      S^T(c), dP^T(c) -> buffer c&1      (issued two chunks ahead)
//   softmax:  P^T, dS^T (bf16) into the same buffer, dS^T into smem tile c&1
//   MMA:      dV += P^T dO, dK += dS^T Q, dQ^T = K^T dS^T (into dP^T's columns)
//   epilogue: dQ^T -> this chunk's Q/dO stage (row-major) -> bulk fp32
//             reduction per token; the stage is then free for chunk c+4.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bwd_main_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                BwdParams p)
{
    using SM = BwdSmem<D>;
    constexpr int kS = SM::kStages;
    constexpr uint32_t kKV = SM::kKV, kHalf = SM::kHalf;
    constexpr int kSlabs = D / 64;
    extern __shared__ __align__(1024) uint8_t smem[];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const RangeItem item = range_item((int)blockIdx.x, p.nblk, p.RB, p.per_group, p.ptr, p.off);
    const int n = item.n, bg = item.bg;
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int G = 1 << p.lgG;
    const int count = item.count;
    const uint32_t code0 = kStTimeoutBase + kKidBwd * 16;
    if (count <= 0) return;   // accumulators start at zero: nothing to add
    if ((smem_u32(smem) & 1023u) != 0u) {   // the swizzled tiles need a 1024-byte aligned base
        if (threadIdx.x == 0) atomicCAS(p.status, 0u, code0 + 15);
        return;
    }
    const int32_t* toks = p.tok + (int64_t)bg * p.T * p.topk + item.beg;
    const int nchunks = (count + p.tpc - 1) / p.tpc;

    uint8_t* k_tile = smem + SM::kK;
    uint8_t* v_tile = smem + SM::kV;
    uint64_t* bars = (uint64_t*)(smem + SM::kBars);
    uint64_t* kv_full = bars;
    uint64_t* st_full = bars + 1;           // [kS] producers -> MMA
    uint64_t* st_empty = st_full + kS;      // [kS] dQ epilogue -> producers
    uint64_t* s_full = st_empty + kS;       // [2] MMA -> softmax
    uint64_t* p_full = s_full + 2;          // [2] softmax -> MMA
    uint64_t* ds_empty = p_full + 2;        // [2] MMA (dQ^T read dS tile) -> softmax
    uint64_t* dq_full = ds_empty + 2;       // [2] MMA -> dQ epilogue
    uint64_t* dq_empty = dq_full + 2;       // [2] dQ epilogue (TMEM drained) -> MMA
    uint64_t* kv_done = dq_empty + 2;
    uint64_t* fin = kv_done + 1;
    uint32_t* tmem_hold = (uint32_t*)(bars + SM::kNumBars);
    volatile uint32_t* abort_flag = tmem_hold + 1;
    const WaitCtx wc{p.status, abort_flag, MSA_WAIT_LIMIT_NS};

    auto q_stage = [&](int s) { return smem + SM::kStage0 + (uint32_t)s * 2u * kHalf; };
    auto do_stage = [&](int s) { return smem + SM::kStage0 + (uint32_t)s * 2u * kHalf + kHalf; };
    auto ds_tile = [&](int bb) { return smem + SM::kDS + (uint32_t)bb * SM::kDSTile; };
    auto meta_l2 = [&](int s) { return (float*)(smem + SM::kMeta + s * SM::kMetaStage); };
    auto meta_d = [&](int s) { return (float*)(smem + SM::kMeta + s * SM::kMetaStage + 256); };
    auto meta_cm = [&](int s) { return (int8_t*)(smem + SM::kMeta + s * SM::kMetaStage + 512); };

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < kS; ++s) { mbar_init(&st_full[s], 128); mbar_init(&st_empty[s], 1); }
        for (int bb = 0; bb < 2; ++bb) {
            mbar_init(&s_full[bb], 1);
            mbar_init(&p_full[bb], 128);
            mbar_init(&ds_empty[bb], 1);
            mbar_init(&dq_full[bb], 1);
            mbar_init(&dq_empty[bb], 128);
        }
        mbar_init(kv_done, 1);
        mbar_init(fin, 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 1) { tmem_alloc(tmem_hold, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_hold;
    // TMEM columns: buffer bb at bb*128: S^T/P^T [0,64), dP^T/dS^T/dQ^T [64,128);
    // dV at 256, dK at 256 + D.
    auto tS = [&](int bb) { return tmem + (uint32_t)bb * 128u; };
    auto tdP = [&](int bb) { return tmem + (uint32_t)bb * 128u + 64u; };
    const uint32_t tdV = tmem + 256u, tdK = tmem + 256u + D;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_arrive_expect_tx(kv_full, 2 * kKV);
            for (int s = 0; s < kSlabs; ++s) {
                tma_load_4d(k_tile + s * 16384, &tm_k, kv_full, s * 64, g, n * 128, b);
                tma_load_4d(v_tile + s * 16384, &tm_v, kv_full, s * 64, g, n * 128, b);
            }
            mbar_drain(kv_full, 0);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idSS = idesc_bf16(128, 64, false, false);    // S^T, dP^T
            constexpr uint32_t idKV = idesc_bf16(128, D, false, true);      // dV, dK (A in TMEM)
            constexpr uint32_t idQT = idesc_bf16(128, 64, true, true);      // dQ^T (M = d, padded to 128)
            const uint32_t ka = smem_u32(k_tile), va = smem_u32(v_tile);
            auto issue_pre = [&](int c) -> bool {   // S^T(c), dP^T(c)
                const int s = c % kS, bb = c & 1;
                if (!mbar_wait(&st_full[s], (uint32_t)(c / kS) & 1u, wc, code0 + 1)) return false;
                if (c >= 2 && !mbar_wait(&dq_empty[bb], (uint32_t)((c - 2) >> 1) & 1u, wc, code0 + 2))
                    return false;
                tc_fence_after();
                const uint32_t qa = smem_u32(q_stage(s)), oa = smem_u32(do_stage(s));
                // S^T and dP^T are independent accumulation chains: interleaving
                // their K-steps keeps more MMAs in flight than one chain at a time
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    umma_ss(tS(bb), desc_kmajor(ka, 128, kk * 16), desc_kmajor(qa, 64, kk * 16), idSS,
                            kk > 0 ? 1u : 0u);
                    umma_ss(tdP(bb), desc_kmajor(va, 128, kk * 16), desc_kmajor(oa, 64, kk * 16), idSS,
                            kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[bb]);
                return true;
            };
            bool ok = mbar_wait(kv_full, 0, wc, code0 + 0);
            if (ok && nchunks > 0) ok = issue_pre(0);
            if (ok && nchunks > 1) ok = issue_pre(1);
            for (int c = 0; ok && c < nchunks; ++c) {
                const int s = c % kS, bb = c & 1;
                if (!mbar_wait(&p_full[bb], (uint32_t)(c >> 1) & 1u, wc, code0 + 3)) break;
                tc_fence_after();
                const uint32_t qa = smem_u32(q_stage(s)), oa = smem_u32(do_stage(s));
                const uint32_t dsa = smem_u32(ds_tile(bb));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {   // K = 64 rows; dV and dK chains interleaved
                    umma_ts(tdV, tS(bb) + kk * 8, desc_mnmajor(oa, 64, kk * 16), idKV,
                            (c > 0 || kk > 0) ? 1u : 0u);
                    umma_ts(tdK, tdP(bb) + kk * 8, desc_mnmajor(qa, 64, kk * 16), idKV,
                            (c > 0 || kk > 0) ? 1u : 0u);
                }
                // dQ^T = K^T dS^T over the 128 keys; with d = 64 the second half
                // of the M = 128 tile reads the V tile and lands in TMEM lanes
                // nobody reads.
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ss(tdP(bb), desc_mnmajor(ka, 128, kk * 16), desc_mnmajor(dsa, 128, kk * 16), idQT,
                            kk > 0 ? 1u : 0u);
                umma_commit(&ds_empty[bb]);
                umma_commit(&dq_full[bb]);
                if (c + 2 < nchunks) ok = issue_pre(c + 2);
            }
            umma_commit(kv_done);
            umma_commit(fin);
            mbar_drain(fin, 0);
        }
    } else if (warp < 6) {
        // ---------------- gather Q, dO (64 rows) and per-row metadata ----------------
        const int tid = threadIdx.x - 64;
        constexpr int kPieces = 64 * D / 8;
        constexpr int kRowPieces = D / 8;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kS;
            const uint32_t su = (uint32_t)(c / kS);
            if (su > 0 && !mbar_wait(&st_empty[s], (su - 1) & 1u, wc, code0 + 4)) break;
            const uint32_t qs = smem_u32(q_stage(s)), os = smem_u32(do_stage(s));
#pragma unroll 4
            for (int it = 0; it < kPieces / 128; ++it) {
                const int piece = it * 128 + tid;
                const int row = piece / kRowPieces, ch = piece % kRowPieces;
                const int t = row >> p.lgG, hh = row & (G - 1);
                const int jj = c * p.tpc + t;
                const bool valid = jj < count;
                const int i = valid ? toks[jj] : 0;
                const int64_t off = (((int64_t)b * p.T + i) * p.Hq + g * G + hh) * D + ch * 8;
                const uint32_t dst = sw128_offset(row, ch & 7, ch >> 3, 64);
                cp_async_16(qs + dst, p.q + off, valid ? 16u : 0u);
                cp_async_16(os + dst, p.dout + off, valid ? 16u : 0u);
            }
            if (tid < 64) {
                const int row = tid;
                const int t = row >> p.lgG, hh = row & (G - 1), h = g * G + hh;
                const int jj = c * p.tpc + t;
                const bool valid = jj < count;
                const int i = valid ? toks[jj] : 0;
                const int64_t lrow = ((int64_t)b * p.Hq + h) * p.T + i;
                meta_l2(s)[row] = valid ? p.lse[lrow] * kLog2e : 0.f;
                meta_d(s)[row] = valid ? p.dsum[lrow] : 0.f;
                meta_cm(s)[row] = (int8_t)(valid ? (((i >> 7) == n) ? (i & 127) : 127) : -1);
            }
            cp_async_commit();
            cp_async_wait<0>();
            fence_proxy_async_smem();
            mbar_arrive(&st_full[s]);
        }
        cp_async_wait<0>();
    } else if (warp < 10) {
        // ---------------- P^T, dS^T (one TMEM lane = one key) ----------------
        const int jl = ((warp & 3) << 5) | lane;   // key within the block
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kS, bb = c & 1;
            bool ok = mbar_wait(&s_full[bb], (uint32_t)(c >> 1) & 1u, wc, code0 + 5);
            if (ok && c >= 2) ok = mbar_wait(&ds_empty[bb], (uint32_t)((c - 2) >> 1) & 1u, wc, code0 + 6);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const float* L2 = meta_l2(s);
            const float* Dv = meta_d(s);
            const int8_t* cm = meta_cm(s);
            const uint32_t aS = tmem_addr(tS(bb), lane_base, 0), aP = tmem_addr(tdP(bb), lane_base, 0);
            const uint32_t dsa = smem_u32(ds_tile(bb));
#pragma unroll
            for (int piece = 0; piece < 2; ++piece) {
                uint32_t sv[32], dv[32], pk[16], dk[16];
                tmem_ld32(aS + piece * 32, sv);
                tmem_ld32(aP + piece * 32, dv);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int r0 = piece * 32 + 2 * e, r1 = r0 + 1;
                    const float p0 = jl <= (int)cm[r0]
                                         ? ex2_approx(fmaf(__uint_as_float(sv[2 * e]), p.c1, -L2[r0]))
                                         : 0.f;
                    const float p1 = jl <= (int)cm[r1]
                                         ? ex2_approx(fmaf(__uint_as_float(sv[2 * e + 1]), p.c1, -L2[r1]))
                                         : 0.f;
                    const float d0 = p0 * (__uint_as_float(dv[2 * e]) - Dv[r0]) * p.scale;
                    const float d1 = p1 * (__uint_as_float(dv[2 * e + 1]) - Dv[r1]) * p.scale;
                    pk[e] = pack_bf16x2(p0, p1);
                    dk[e] = pack_bf16x2(d0, d1);
                }
                tmem_st16(aS + piece * 16, pk);   // P^T over S^T columns already read
                tmem_st16(aP + piece * 16, dk);   // dS^T over dP^T columns already read
                // dS^T row jl (rows piece*32 .. +31) into the MN-major dS tile
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    const uint32_t addr = dsa + sw128_offset((uint32_t)jl, (uint32_t)(piece * 4 + qd), 0, 128);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dk[4 * qd]),
                                 "r"(dk[4 * qd + 1]), "r"(dk[4 * qd + 2]), "r"(dk[4 * qd + 3])
                                 : "memory");
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&p_full[bb]);
        }
    } else {
        // ---------------- dQ partials out; dK, dV partials at the end ----------------
        const int r = ((warp & 3) << 5) | lane;    // TMEM lane = head-dim index of dQ^T
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
        const int tid = threadIdx.x - 320;
        const uint32_t tok_bytes = (uint32_t)G * D * 4u;
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kS, bb = c & 1;
            ok = bar_and_sync(1, 128, mbar_wait(&dq_full[bb], (uint32_t)(c >> 1) & 1u, wc, code0 + 7));
            if (!ok) break;   // all four warps leave together: none is left at a barrier below
            tc_fence_after();
            // dQ^T[r][row] for the chunk's 64 rows -> row-major staging in this
            // chunk's Q/dO stage (32 consecutive floats per warp store)
            const uint32_t stg = smem_u32(q_stage(s));
            uint32_t v[64];
            tmem_ld32(tmem_addr(tdP(bb), lane_base, 0), v);
            tmem_ld32(tmem_addr(tdP(bb), lane_base, 32), v + 32);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&dq_empty[bb]);     // TMEM columns free for chunk c+2
            if (r < D) {
#pragma unroll
                for (int e = 0; e < 64; ++e)
                    asm volatile("st.shared.b32 [%0], %1;" ::"r"(stg + ((uint32_t)e * D + (uint32_t)r) * 4u),
                                 "r"(v[e])
                                 : "memory");
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            const int ntok = min(p.tpc, count - c * p.tpc);
            for (int t = tid; t < ntok; t += 128) {
                const int i = toks[c * p.tpc + t];
                asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
                                 p.dqacc + (((int64_t)b * p.T + i) * p.Hq + g * G) * D),
                             "r"(stg + (uint32_t)t * tok_bytes), "r"(tok_bytes)
                             : "memory");
            }
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            named_bar_sync(1, 128);
            if (tid == 0) mbar_arrive(&st_empty[s]);
        }
        if (ok) ok = mbar_wait(kv_done, 0, wc, code0 + 8);
        if (__all_sync(0xffffffffu, ok)) {
            // This item's dK, dV partials (lane = key) -> padded staging in the
            // now idle stage and dS area -> one bulk fp32 reduction per key row.
            tc_fence_after();
            const uint32_t row_stride = D * 4u + 16u;
            const uint32_t stg = smem_u32(smem + SM::kStage0);
            const int j = n * 128 + r;   // this lane's key
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t ta = tmem_addr(which == 0 ? tdV : tdK, lane_base, 0);
                const uint32_t row = stg + (uint32_t)which * 128u * row_stride + (uint32_t)r * row_stride;
#pragma unroll
                for (int piece = 0; piece < D / 32; ++piece) {
                    uint32_t w[32];
                    tmem_ld32(ta + piece * 32, w);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + (piece * 32 + 4 * e) * 4),
                                     "r"(w[4 * e]), "r"(w[4 * e + 1]), "r"(w[4 * e + 2]), "r"(w[4 * e + 3])
                                     : "memory");
                }
            }
            fence_proxy_async_smem();
            if (j < p.T) {
                const int64_t off = (((int64_t)b * p.T + j) * p.Hkv + g) * D;
#pragma unroll
                for (int which = 0; which < 2; ++which) {
                    float* dst = (which == 0 ? p.dvacc : p.dkacc) + off;
                    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
                                 "r"(stg + (uint32_t)which * 128u * row_stride + (uint32_t)r * row_stride),
                                 "r"((uint32_t)D * 4u)
                                 : "memory");
                }
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// D_i = dO_i . O_i per query row (bf16 inputs, fp32 sum); D/8 lanes per row.
template <int D>
__global__ void __launch_bounds__(256) bwd_dsum_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout, int B, int T,
                                                       int Hq, float* __restrict__ dsum)
{
    constexpr int LPR = D / 8;
    const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = gt / LPR;
    const int sub = (int)(gt % LPR);
    const bool ok = row < (int64_t)B * T * Hq;
    float s = 0.f;
    if (ok) {
        const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + sub * 8);
        const uint4 c = *reinterpret_cast<const uint4*>(dout + row * D + sub * 8);
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&c);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(a2[e]), y = __bfloat1622float2(c2[e]);
            s = fmaf(x.x, y.x, s);
            s = fmaf(x.y, y.y, s);
        }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (ok && sub == 0) {
        const int h = (int)(row % Hq);
        const int64_t bi = row / Hq;
        const int i = (int)(bi % T), b = (int)(bi / T);
        dsum[((int64_t)b * Hq + h) * T + i] = s;
    }
}

// fp32 dQ accumulator -> bf16, 8 elements per thread.
__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(const float* __restrict__ acc,
                                                             __nv_bfloat16* __restrict__ dq, int64_t n8)
{
    const int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= n8) return;
    const float4 a = *reinterpret_cast<const float4*>(acc + x * 8);
    const float4 c = *reinterpret_cast<const float4*>(acc + x * 8 + 4);
    uint4 u;
    u.x = pack_bf16x2(a.x, a.y);
    u.y = pack_bf16x2(a.z, a.w);
    u.z = pack_bf16x2(c.x, c.y);
    u.w = pack_bf16x2(c.z, c.w);
    *reinterpret_cast<uint4*>(dq + x * 8) = u;
}

template <int D>
cudaError_t launch_bwd_d(const Problem& pr, const void* q, const void* dout, const CUtensorMap& tm_k,
                         const CUtensorMap& tm_v, const void* o, const float* lse, void* dq, void* dk,
                         void* dv, void* ws, const WsLayout& L, cudaStream_t st)
{
    uint8_t* w = (uint8_t*)ws;
    float* dsum = (float*)(w + L.dsum);
    float* dqacc = (float*)(w + L.dqacc);
    float* dkacc = (float*)(w + L.dkacc);
    float* dvacc = (float*)(w + L.dvacc);
    const size_t kv_elems = (size_t)pr.B * pr.T * pr.Hkv * D;
    cudaError_t e;
    if ((e = cudaMemsetAsync(dqacc, 0, sizeof(float) * (size_t)pr.rows_q() * D, st)) != cudaSuccess)
        return e;
    if ((e = cudaMemsetAsync(dkacc, 0, sizeof(float) * kv_elems, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dvacc, 0, sizeof(float) * kv_elems, st)) != cudaSuccess) return e;
    const int64_t th = pr.rows_q() * (D / 8);
    bwd_dsum_kernel<D><<<(unsigned)((th + 255) / 256), 256, 0, st>>>(
        (const __nv_bfloat16*)o, (const __nv_bfloat16*)dout, pr.B, pr.T, pr.Hq, dsum);

    BwdParams p;
    p.B = pr.B; p.T = pr.T; p.Hq = pr.Hq; p.Hkv = pr.Hkv;
    p.lgG = 31 - __builtin_clz((unsigned)pr.G);
    p.tpc = 64 / pr.G; p.nblk = pr.nblk; p.topk = pr.topk;   // 64-row chunks
    p.c1 = pr.scale * kLog2e;
    p.scale = pr.scale;
    p.q = (const __nv_bfloat16*)q;
    p.dout = (const __nv_bfloat16*)dout;
    p.lse = lse;
    p.dsum = dsum;
    p.ptr = (const int32_t*)(w + L.ptr);
    p.off = (const int32_t*)(w + L.cnt);
    p.tok = (const int32_t*)(w + L.tok);
    p.dqacc = dqacc;
    p.dkacc = dkacc;
    p.dvacc = dvacc;
    p.status = (uint32_t*)(w + L.status);
    p.RB = range_blocks(pr);
    p.per_group = range_items_per_group(pr.nblk, p.RB);
    const size_t smem = BwdSmem<D>::kTotal;
    if ((e = cudaFuncSetAttribute(bwd_main_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess)
        return e;
    trace_begin(kTraceBwdMain, st);
    bwd_main_kernel<D><<<(unsigned)(p.per_group * pr.B * pr.Hkv), kThreads, smem, st>>>(tm_k, tm_v, p);
    trace_end(kTraceBwdMain, st);
    const int64_t n8 = pr.rows_q() * D / 8;
    bwd_dq_convert_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(dqacc, (__nv_bfloat16*)dq, n8);
    const int64_t k8 = (int64_t)kv_elems / 8;
    bwd_dq_convert_kernel<<<(unsigned)((k8 + 255) / 256), 256, 0, st>>>(dkacc, (__nv_bfloat16*)dk, k8);
    bwd_dq_convert_kernel<<<(unsigned)((k8 + 255) / 256), 256, 0, st>>>(dvacc, (__nv_bfloat16*)dv, k8);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(const Problem& pr, const void* q, const void* dout, const CUtensorMap& tm_k,
                       const CUtensorMap& tm_v, const void* o, const float* lse, void* dq, void* dk,
                       void* dv, void* ws, const WsLayout& L, cudaStream_t st)
{
    if (pr.d == 64) return launch_bwd_d<64>(pr, q, dout, tm_k, tm_v, o, lse, dq, dk, dv, ws, L, st);
    return launch_bwd_d<128>(pr, q, dout, tm_k, tm_v, o, lse, dq, dk, dv, ws, L, st);
}

}  // namespace msa
