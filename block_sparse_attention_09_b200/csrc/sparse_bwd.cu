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
// shared memory and dK, dV as fp32 accumulators in TMEM for the whole work
// item, so dK/dV need no atomics.  The queries that selected the block are
// gathered with cp.async in chunks of 128 rows (128/G tokens x G heads) into
// a 2-stage ring.  Per chunk, in the transposed orientation so that one TMEM
// lane is one key, and with every MMA 128 wide (an M=128 tcgen05 MMA costs
// about the same per instruction at N=64 as at N=128):
//   S^T = K Q^T -> TMEM [0,128),  dP^T = V dO^T -> TMEM [128,256)
//   softmax warps: P^T (bf16) over the S^T columns already read, and
//                  dS^T = P^T (dP^T scale - D scale) (bf16) into a shared-memory tile
//   dV += P^T dO (A from TMEM), dK += dS^T Q (A = the dS tile, K-major),
//   dQ^T = K^T dS^T (B = the same tile, MN-major) -> TMEM [128,256)
//   dQ^T -> row-major staging in the chunk's Q/dO stage, a quarter (32 rows)
//   at a time -> one bulk fp32 reduction per token into a global accumulator,
//   issued by warp 0 so that the staging warps never wait on the reduction.
// TMEM holds one chunk at a time (S^T, dP^T, dV, dK fill all 512 columns);
// S^T of the next chunk is issued right behind the current chunk's MMAs and
// dP^T once the dQ^T columns have been read out.
#include <math.h>

#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kWarps = 18;   // w0 TMA(K,V), dQ reductions | w1 MMA | w2-9 softmax | w10-13 gather | w14-17 dQ, dK/dV
constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
    int B, T, Hq, Hkv, lgG, tpc, nblk, topk;
    int RB, qb0, per_group;   // query blocks per range; first query block; work items per (b, group)
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
    static constexpr uint32_t kKV = 128u * D * 2u;              // one K or V tile
    static constexpr uint32_t kHalf = 128u * D * 2u;            // Q or dO of one 128-row chunk
    static constexpr uint32_t kK = 0, kV = kKV;                 // V right after K (d = 64 dQ^T reads on)
    static constexpr uint32_t kStage0 = 2 * kKV;                // stage s: Q at s*2*kHalf, dO after it
    static constexpr uint32_t kDS = kStage0 + 2 * 2 * kHalf;    // dS^T tile: 128 keys x 128 rows bf16
    static constexpr uint32_t kDSBytes = 128u * 128u * 2u;
    static constexpr uint32_t kMeta = kDS + kDSBytes;           // per stage {L2[128], D*scale[128], cm[128], flag}
    static constexpr uint32_t kMetaStage = 128 * 4 * 2 + 128 + 16;
    static constexpr uint32_t kBars = kMeta + 2 * kMetaStage;
    static constexpr uint32_t kNumBars = 1 + 2 + 2 + 5 + 8;
    static constexpr uint32_t kTotal = kBars + kNumBars * 8 + 8;
    static_assert(kTotal <= 232448, "shared memory per CTA");
    static_assert(2 * 128 * (D * 4 + 16) <= kMeta - kStage0, "dK/dV staging must fit the stage and dS area");
    static_assert(128u * D * 4u <= 2 * kHalf, "dQ staging must fit one stage");
};

// Work per item: chunks c of 128 query rows, token-major (row = t*G + hh).
template <int D>
__global__ void __launch_bounds__(kWarps * 32, 1)
bwd_main_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                BwdParams p)
{
    using SM = BwdSmem<D>;
    constexpr uint32_t kKV = SM::kKV, kHalf = SM::kHalf;
    constexpr int kSlabs = D / 64;
    extern __shared__ __align__(1024) uint8_t smem[];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const RangeItem item = range_item((int)blockIdx.x, p.nblk, p.RB, p.qb0, p.per_group, p.ptr, p.off);
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
    uint64_t* st_full = bars + 1;           // [2] gather -> MMA, softmax
    uint64_t* st_empty = st_full + 2;       // [2] dQ epilogue (staging read) -> gather
    uint64_t* s_full = st_empty + 2;        // MMA -> softmax (S^T, dP^T; earlier MMAs done)
    uint64_t* p_full = s_full + 1;          // softmax -> MMA (P^T in TMEM, dS^T in smem)
    uint64_t* dq_full = p_full + 1;         // MMA -> dQ epilogue (every MMA of the chunk done)
    uint64_t* dq_drained = dq_full + 1;     // dQ epilogue (TMEM read) -> MMA
    uint64_t* fin = dq_drained + 1;
    uint64_t* stg_full = fin + 1;           // [2][4] dQ epilogue (quarter staged) -> warp 0
    uint32_t* tmem_hold = (uint32_t*)(bars + SM::kNumBars);
    volatile uint32_t* abort_flag = tmem_hold + 1;
    const WaitCtx wc{p.status, abort_flag, MSA_WAIT_LIMIT_NS};

    auto q_stage = [&](int s) { return smem + SM::kStage0 + (uint32_t)s * 2u * kHalf; };
    auto do_stage = [&](int s) { return smem + SM::kStage0 + (uint32_t)s * 2u * kHalf + kHalf; };
    uint8_t* ds_tile = smem + SM::kDS;
    auto meta_l2 = [&](int s) { return (float*)(smem + SM::kMeta + s * SM::kMetaStage); };
    auto meta_d = [&](int s) { return (float*)(smem + SM::kMeta + s * SM::kMetaStage + 512); };
    auto meta_cm = [&](int s) { return (int8_t*)(smem + SM::kMeta + s * SM::kMetaStage + 1024); };
    auto meta_flag = [&](int s) { return (int*)(smem + SM::kMeta + s * SM::kMetaStage + 1152); };

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < 2; ++s) { mbar_init(&st_full[s], 128); mbar_init(&st_empty[s], 1); }
        mbar_init(s_full, 1);
        mbar_init(p_full, 256);
        mbar_init(dq_full, 1);
        mbar_init(dq_drained, 128);
        mbar_init(fin, 1);
        for (int x = 0; x < 8; ++x) mbar_init(&stg_full[x], 128);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 1) { tmem_alloc(tmem_hold, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_hold;
    // TMEM columns: S^T / P^T [0,128), dP^T / dQ^T [128,256), dV at 256, dK at 256 + D.
    const uint32_t tS = tmem, tdP = tmem + 128u;
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
        __syncwarp();
        // ---------------- dQ bulk reductions ----------------
        // Quarter qq of chunk c holds tokens [qq*qt, qq*qt + qt) of the chunk;
        // lane l reduces token qq*qt + l.  Stage sets alternate with the chunk
        // parity, so a set is reused only after this warp released its stage.
        const int qt = p.tpc >> 2;
        const uint32_t tok_bytes = (uint32_t)G * D * 4u;
        int tq[4];
        auto load_tokens = [&](int c) {
            const int ntok = min(p.tpc, count - c * p.tpc);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const int t = qq * qt + lane;
                tq[qq] = (lane < qt && t < ntok) ? __ldg(toks + c * p.tpc + t) : -1;
            }
        };
        load_tokens(0);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const uint32_t stg = smem_u32(q_stage(s));
            bool ok = true;
            bool issued = false;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                ok = mbar_wait(&stg_full[s * 4 + qq], (uint32_t)(c >> 1) & 1u, wc, code0 + 9);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                if (tq[qq] >= 0) {
                    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
                                     p.dqacc + (((int64_t)b * p.T + tq[qq]) * p.Hq + g * G) * D),
                                 "r"(stg + (uint32_t)(qq * qt + lane) * tok_bytes), "r"(tok_bytes)
                                 : "memory");
                    issued = true;
                }
            }
            if (issued) asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            if (!ok) break;
            if (c + 1 < nchunks) load_tokens(c + 1);
            if (issued) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&st_empty[s]);   // staging read: the stage may be refilled
        }
        // the shared-memory source must have been read before the CTA exits;
        // the global side completes on its own
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 128, false, false);    // S^T, dP^T (N = 128 rows)
            constexpr uint32_t idKV = idesc_bf16(128, D, false, true);      // dV, dK (N = d)
            constexpr uint32_t idQT = idesc_bf16(128, 128, true, true);     // dQ^T (M = d, padded to 128)
            const uint32_t ka = smem_u32(k_tile), va = smem_u32(v_tile), dsa = smem_u32(ds_tile);
            bool ok = mbar_wait(kv_full, 0, wc, code0 + 0);
            for (int c = 0; ok && c < nchunks; ++c) {
                const int s = c & 1;
                if (!mbar_wait(&st_full[s], (uint32_t)(c >> 1) & 1u, wc, code0 + 1)) break;
                tc_fence_after();
                const uint32_t qa = smem_u32(q_stage(s)), oa = smem_u32(do_stage(s));
                // S^T(c): its columns held P^T(c-1), which the dV MMAs issued
                // before this point have consumed (MMAs run in issue order)
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    umma_ss(tS, desc_kmajor(ka, 128, kk * 16), desc_kmajor(qa, 128, kk * 16), idS,
                            kk > 0 ? 1u : 0u);
                // dP^T(c) overwrites dQ^T(c-1): wait until it has been read out
                if (c > 0 && !mbar_wait(dq_drained, (uint32_t)(c - 1) & 1u, wc, code0 + 2)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    umma_ss(tdP, desc_kmajor(va, 128, kk * 16), desc_kmajor(oa, 128, kk * 16), idS,
                            kk > 0 ? 1u : 0u);
                umma_commit(s_full);
                if (!mbar_wait(p_full, (uint32_t)c & 1u, wc, code0 + 3)) break;
                tc_fence_after();
                // dV, dK (K = 128 rows) and dQ^T (K = 128 keys): three independent
                // accumulation chains, interleaved
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t pcol = kk < 4 ? (uint32_t)kk * 8u : 64u + (uint32_t)(kk - 4) * 8u;
                    umma_ts(tdV, tS + pcol, desc_mnmajor(oa, 128, kk * 16), idKV, (c > 0 || kk > 0) ? 1u : 0u);
                    umma_ss(tdK, desc_kmajor(dsa, 128, kk * 16), desc_mnmajor(qa, 128, kk * 16), idKV,
                            (c > 0 || kk > 0) ? 1u : 0u);
                    umma_ss(tdP, desc_mnmajor(ka, 128, kk * 16), desc_mnmajor(dsa, 128, kk * 16), idQT,
                            kk > 0 ? 1u : 0u);
                }
                umma_commit(dq_full);
            }
            umma_commit(fin);
            mbar_drain(fin, 0);
        }
    } else if (warp < 10) {
        // ---------------- P^T, dS^T (one TMEM lane = one key) ----------------
        // Two warps per TMEM lane quarter: warp half hf takes rows [64 hf, 64 hf + 64).
        const int qd4 = warp & 3, hf = (warp - 2) >> 2;
        const int jl = (qd4 << 5) | lane;   // key within the block
        const uint32_t lane_base = (uint32_t)(qd4 * 32);
        const uint32_t dsa = smem_u32(ds_tile);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            // s_full(c) also means dK(c-1) and dQ^T(c-1) have read the dS tile;
            // st_full (long complete by then) orders the gather's metadata stores
            bool ok = mbar_wait(s_full, (uint32_t)c & 1u, wc, code0 + 5);
            if (ok) ok = mbar_wait(&st_full[s], (uint32_t)(c >> 1) & 1u, wc, code0 + 6);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const float* L2 = meta_l2(s);
            const float* Dv = meta_d(s);
            const int8_t* cm = meta_cm(s);
            const bool masked = *(volatile int*)meta_flag(s) != 0;   // chunk holds block-n queries
#pragma unroll
            for (int pp = 0; pp < 2; ++pp) {
                const int piece = 2 * hf + pp;   // rows piece*32 .. +31
                uint32_t sv[32], dv[32], pk[16], dk[16];
                tmem_ld32(tmem_addr(tS, lane_base, (uint32_t)piece * 32u), sv);
                tmem_ld32(tmem_addr(tdP, lane_base, (uint32_t)piece * 32u), dv);
                tmem_ld_wait();
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const int r0 = piece * 32 + 4 * e4;
                    const float4 l4 = *reinterpret_cast<const float4*>(L2 + r0);
                    const float4 d4 = *reinterpret_cast<const float4*>(Dv + r0);
                    float pr[4];
                    pr[0] = ex2_approx(fmaf(__uint_as_float(sv[4 * e4 + 0]), p.c1, -l4.x));
                    pr[1] = ex2_approx(fmaf(__uint_as_float(sv[4 * e4 + 1]), p.c1, -l4.y));
                    pr[2] = ex2_approx(fmaf(__uint_as_float(sv[4 * e4 + 2]), p.c1, -l4.z));
                    pr[3] = ex2_approx(fmaf(__uint_as_float(sv[4 * e4 + 3]), p.c1, -l4.w));
                    if (masked) {
                        const uint32_t c4 = *reinterpret_cast<const uint32_t*>(cm + r0);
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if (jl > (int)(int8_t)(c4 >> (8 * u))) pr[u] = 0.f;
                    }
                    // dS = P (dP - D) scale, as P (dP scale - D scale)
                    const float s0 = pr[0] * fmaf(__uint_as_float(dv[4 * e4 + 0]), p.scale, -d4.x);
                    const float s1 = pr[1] * fmaf(__uint_as_float(dv[4 * e4 + 1]), p.scale, -d4.y);
                    const float s2 = pr[2] * fmaf(__uint_as_float(dv[4 * e4 + 2]), p.scale, -d4.z);
                    const float s3 = pr[3] * fmaf(__uint_as_float(dv[4 * e4 + 3]), p.scale, -d4.w);
                    pk[2 * e4] = pack_bf16x2(pr[0], pr[1]);
                    pk[2 * e4 + 1] = pack_bf16x2(pr[2], pr[3]);
                    dk[2 * e4] = pack_bf16x2(s0, s1);
                    dk[2 * e4 + 1] = pack_bf16x2(s2, s3);
                }
                // P^T rows piece*32.. over S^T columns this warp has already read
                tmem_st16(tmem_addr(tS, lane_base, (uint32_t)(64 * hf + 16 * pp)), pk);
                // dS^T row jl, query rows piece*32 .. +31 (slab piece/2 of the tile)
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    const uint32_t addr =
                        dsa + sw128_offset((uint32_t)jl, (uint32_t)((piece & 1) * 4 + qd), (uint32_t)(piece >> 1), 128);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dk[4 * qd]),
                                 "r"(dk[4 * qd + 1]), "r"(dk[4 * qd + 2]), "r"(dk[4 * qd + 3])
                                 : "memory");
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(p_full);
        }
    } else if (warp < 14) {
        // ---------------- gather Q, dO (128 rows) and per-row metadata ----------------
        // Thread tid copies 16-byte column ch of rows r0, r0 + kRowStep, ...:
        // two neighbouring rows per warp and instruction, each row whole.  The
        // next chunk's token ids and metadata are loaded while this chunk's
        // copies are in flight.
        const int tid = threadIdx.x - 320;
        constexpr int kRowPieces = D / 8;
        constexpr int kRowStep = 128 / kRowPieces;
        const int ch = tid % kRowPieces, r0 = tid / kRowPieces;
        int tk[kRowPieces];          // token of each of this thread's rows (-1: past the end)
        int m_tok = -1, m_tok_next = -1;   // token of metadata row tid: this chunk, the next
        float m_l2 = 0.f, m_d = 0.f;
        auto row_tokens = [&](int c) {
#pragma unroll
            for (int it = 0; it < kRowPieces; ++it) {
                const int jj = c * p.tpc + ((r0 + it * kRowStep) >> p.lgG);
                tk[it] = jj < count ? __ldg(toks + jj) : -1;
            }
        };
        auto meta_token = [&](int c) {
            const int jj = c * p.tpc + (tid >> p.lgG);
            return (c < nchunks && jj < count) ? __ldg(toks + jj) : -1;
        };
        auto meta_values = [&]() {   // for m_tok, loaded one chunk before its use
            if (m_tok >= 0) {
                const int64_t lrow = ((int64_t)b * p.Hq + g * G + (tid & (G - 1))) * p.T + m_tok;
                m_l2 = __ldg(p.lse + lrow) * kLog2e;
                m_d = __ldg(p.dsum + lrow) * p.scale;
            } else {
                m_l2 = 0.f;
                m_d = 0.f;
            }
        };
        row_tokens(0);
        m_tok = meta_token(0);
        meta_values();
        m_tok_next = meta_token(1);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const uint32_t su = (uint32_t)(c >> 1);
            if (su > 0 && !mbar_wait(&st_empty[s], (su - 1) & 1u, wc, code0 + 4)) break;
            const uint32_t qs = smem_u32(q_stage(s)), os = smem_u32(do_stage(s));
#pragma unroll
            for (int it = 0; it < kRowPieces; ++it) {
                const int row = r0 + it * kRowStep;
                const bool valid = tk[it] >= 0;
                const int64_t off =
                    (((int64_t)b * p.T + (valid ? tk[it] : 0)) * p.Hq + g * G + (row & (G - 1))) * D + ch * 8;
                const uint32_t dst = sw128_offset((uint32_t)row, (uint32_t)(ch & 7), (uint32_t)(ch >> 3), 128);
                cp_async_16(qs + dst, p.q + off, valid ? 16u : 0u);
                cp_async_16(os + dst, p.dout + off, valid ? 16u : 0u);
            }
            cp_async_commit();
            {
                // rows past the item's end read as zeros with L2 = D = 0: their P is
                // finite and meets only zero dO, and dP - D = 0, so they add nothing
                const bool diag = m_tok >= 0 && (m_tok >> 7) == n;
                meta_l2(s)[tid] = m_l2;
                meta_d(s)[tid] = m_d;
                meta_cm(s)[tid] = (int8_t)(diag ? (m_tok & 127) : 127);
                // token lists are ascending, so block-n queries come first
                if (tid == 0) *meta_flag(s) = diag ? 1 : 0;
            }
            // next chunk: its row tokens, the metadata of its row tid (whose token
            // arrived during this chunk), and the token of the chunk after it
            if (c + 1 < nchunks) {
                row_tokens(c + 1);
                m_tok = m_tok_next;
                meta_values();
                m_tok_next = meta_token(c + 2);
            }
            cp_async_wait<0>();
            fence_proxy_async_smem();
            mbar_arrive(&st_full[s]);
        }
        cp_async_wait<0>();
    } else {
        // ---------------- dQ partials out; dK, dV partials at the end ----------------
        const int r = ((warp & 3) << 5) | lane;    // TMEM lane = head-dim index of dQ^T
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            ok = mbar_wait(dq_full, (uint32_t)c & 1u, wc, code0 + 7);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            // dQ^T[r][row] for the chunk's 128 rows -> row-major staging in this
            // chunk's Q/dO stage (32 consecutive floats per warp store), handed
            // to warp 0 a quarter at a time
            const uint32_t stg = smem_u32(q_stage(s));
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                uint32_t v[32];
                tmem_ld32(tmem_addr(tdP, lane_base, (uint32_t)qq * 32u), v);
                tmem_ld_wait();
                if (qq == 3) {
                    tc_fence_before();
                    mbar_arrive(dq_drained);     // TMEM columns free for dP^T(c+1)
                }
                if (r < D) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        asm volatile("st.shared.b32 [%0], %1;" ::"r"(stg + ((uint32_t)(qq * 32 + e) * D + (uint32_t)r) * 4u),
                                     "r"(v[e])
                                     : "memory");
                }
                fence_proxy_async_smem();
                mbar_arrive(&stg_full[s * 4 + qq]);
            }
        }
        // the dK/dV staging below reuses both stages: wait until warp 0's
        // reductions have read the last chunks' dQ staging
        for (int c = max(0, nchunks - 2); ok && c < nchunks; ++c)
            ok = __all_sync(0xffffffffu, mbar_wait(&st_empty[c & 1], (uint32_t)(c >> 1) & 1u, wc, code0 + 8));
        if (ok) {
            // The last dq_full covers every MMA of the item.  Its dK, dV partials
            // (lane = key) -> padded staging in the now idle stage and dS area ->
            // one bulk fp32 reduction per key row.
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
                asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// D_i = dO_i . O_i per computed query row (rows q0 .. T-1; bf16 inputs, fp32
// sum); D/8 lanes per row.
template <int D, bool Small>
__global__ void __launch_bounds__(256) bwd_dsum_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout, int B, int T,
                                                       int Hq, int q0, float* __restrict__ dsum)
{
    constexpr int LPR = D / 8;
    const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t ar = gt / LPR;
    const int sub = (int)(gt % LPR);
    const bool ok = ar < (int64_t)B * (T - q0) * Hq;
    int b = 0, i = 0, h = 0;
    if (ok) active_coords<Small>(ar, T, Hq, q0, b, i, h);
    const int64_t row = ((int64_t)b * T + i) * Hq + h;
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
    if (ok && sub == 0) dsum[((int64_t)b * Hq + h) * T + i] = s;
}

// fp32 accumulator -> bf16, 8 elements per thread.
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

// The computed rows (q0 .. T-1) of the fp32 dQ accumulator -> bf16 dQ.
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_rows_kernel(const float* __restrict__ acc,
                                                          __nv_bfloat16* __restrict__ dq, int B, int T, int Hq,
                                                          int q0)
{
    constexpr int LPR = D / 8;
    const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t ar = gt / LPR;
    if (ar >= (int64_t)B * (T - q0) * Hq) return;
    const int64_t x = active_row(ar, T, Hq, q0) * D + (gt % LPR) * 8;
    const float4 a = *reinterpret_cast<const float4*>(acc + x);
    const float4 c = *reinterpret_cast<const float4*>(acc + x + 4);
    uint4 u;
    u.x = pack_bf16x2(a.x, a.y);
    u.y = pack_bf16x2(a.z, a.w);
    u.z = pack_bf16x2(c.x, c.y);
    u.w = pack_bf16x2(c.z, c.w);
    *reinterpret_cast<uint4*>(dq + x) = u;
}

template <int D>
cudaError_t launch_bwd_d(const Problem& pr, const void* q, const void* dout, const CUtensorMap& tm_k,
                         const CUtensorMap& tm_v, const void* o, const float* lse, void* dq, void* dk,
                         void* dv, bool dkv_f32, void* ws, const WsLayout& L, cudaStream_t st)
{
    uint8_t* w = (uint8_t*)ws;
    float* dsum = (float*)(w + L.dsum);
    float* dqacc = (float*)(w + L.dqacc);
    // fp32 dK/dV outputs are accumulated in place
    float* dkacc = dkv_f32 ? (float*)dk : (float*)(w + L.dkacc);
    float* dvacc = dkv_f32 ? (float*)dv : (float*)(w + L.dvacc);
    const size_t kv_elems = (size_t)pr.B * pr.T * pr.Hkv * D;
    cudaError_t e;
    if ((e = cudaMemsetAsync(dqacc, 0, sizeof(float) * (size_t)pr.rows_q() * D, st)) != cudaSuccess)
        return e;
    if ((e = cudaMemsetAsync(dkacc, 0, sizeof(float) * kv_elems, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dvacc, 0, sizeof(float) * kv_elems, st)) != cudaSuccess) return e;
    const int64_t th = pr.rows_q_active() * (D / 8);
    if (th < ((int64_t)1 << 31))
        bwd_dsum_kernel<D, true><<<(unsigned)((th + 255) / 256), 256, 0, st>>>(
            (const __nv_bfloat16*)o, (const __nv_bfloat16*)dout, pr.B, pr.T, pr.Hq, pr.q0, dsum);
    else
        bwd_dsum_kernel<D, false><<<(unsigned)((th + 255) / 256), 256, 0, st>>>(
            (const __nv_bfloat16*)o, (const __nv_bfloat16*)dout, pr.B, pr.T, pr.Hq, pr.q0, dsum);
    count_launches(1);

    BwdParams p;
    p.B = pr.B; p.T = pr.T; p.Hq = pr.Hq; p.Hkv = pr.Hkv;
    p.lgG = 31 - __builtin_clz((unsigned)pr.G);
    p.tpc = 128 / pr.G; p.nblk = pr.nblk; p.topk = pr.topk;   // 128-row chunks
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
    p.qb0 = pr.qb0;
    p.per_group = range_items_per_group(pr.nblk, p.RB, pr.qb0);
    const size_t smem = BwdSmem<D>::kTotal;
    if ((e = cudaFuncSetAttribute(bwd_main_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess)
        return e;
    trace_begin(kTraceBwdMain, st);
    bwd_main_kernel<D><<<(unsigned)(p.per_group * pr.B * pr.Hkv), kWarps * 32, smem, st>>>(tm_k, tm_v, p);
    count_launches(1);
    trace_end(kTraceBwdMain, st);
    const int64_t n8 = pr.rows_q_active() * D / 8;
    bwd_dq_rows_kernel<D><<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(dqacc, (__nv_bfloat16*)dq, pr.B, pr.T,
                                                                          pr.Hq, pr.q0);
    count_launches(1);
    if (!dkv_f32) {
        const int64_t k8 = (int64_t)kv_elems / 8;
        bwd_dq_convert_kernel<<<(unsigned)((k8 + 255) / 256), 256, 0, st>>>(dkacc, (__nv_bfloat16*)dk, k8);
        count_launches(1);
        bwd_dq_convert_kernel<<<(unsigned)((k8 + 255) / 256), 256, 0, st>>>(dvacc, (__nv_bfloat16*)dv, k8);
        count_launches(1);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(const Problem& pr, const void* q, const void* dout, const CUtensorMap& tm_k,
                       const CUtensorMap& tm_v, const void* o, const float* lse, void* dq, void* dk,
                       void* dv, bool dkv_f32, void* ws, const WsLayout& L, cudaStream_t st)
{
    if (pr.d == 64) return launch_bwd_d<64>(pr, q, dout, tm_k, tm_v, o, lse, dq, dk, dv, dkv_f32, ws, L, st);
    return launch_bwd_d<128>(pr, q, dout, tm_k, tm_v, o, lse, dq, dk, dv, dkv_f32, ws, L, st);
}

cudaError_t launch_f32_to_bf16(const float* src, void* dst, int64_t n, cudaStream_t st)
{
    const int64_t n8 = n / 8;
    bwd_dq_convert_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(src, (__nv_bfloat16*)dst, n8);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace msa
