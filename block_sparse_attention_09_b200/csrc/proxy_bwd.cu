// Proxy-head gradient: the training signal of the Index Branch.
//
// The pages say only that training passes gradients through the gating
// mechanism (ai-beat post on Flash-MSA training, paragraph 2) and that the
// proxy heads are small trained networks (paragraph 4); "Flash-MSA: Open-Source
// Sparse Attention Kernels Debut" (section "How MSA works") likens MSA to
// DeepSeek's sparse attention, whose indexer is trained to match the main
// attention.  The reading built here: per query row (b, g, i) with selected
// blocks S_i,
//   p_i(n) = (1/G) sum_{h in g} (softmax weight of head h on block n),
//   z_i(n) = pooled proxy score of block n (max over its visible keys),
//   q_i    = softmax over n in S_i of z_i(n),
//   loss_i = KL(p_i || q_i),  d loss_i / d z_i(n) = q_i(n) sum_m p_i(m) - p_i(n),
// and the gradient reaches the proxy query of row i and the argmax key j* of
// each block (the lowest key on ties): dqp_i += dz kp_j*, dkp_j* += dz qp_i.
// The selection itself is fixed (top-k is not differentiable).
//
// Three kernels, all driven by the pair index the forward built (lists of
// the queries that selected block 2p or 2p+1, one entry per query):
//   scores  KV-stationary over (group, query range, pair) items: the proxy
//           scores of each entry's query against the pair's 256 keys on the
//           tensor cores (M = 128 queries, N = 256, K = dp), reduced to z and
//           j* of each selected block in the epilogue;
//   rows    one warp per query row: the row's entries (found from the tile's
//           block masks), p from the block masses the forward kept, q, the
//           loss, dz, and dqp (a gather of the argmax proxy keys);
//   keys    one CTA per (group, pair): dkp of the pair's 256 keys from all of
//           its entries, accumulated in shared memory.
#include <math.h>

#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kScThreads = 320;   // w0 TMA | w1 MMA | w2-5 gather | w6-9 epilogue
constexpr uint32_t kRowBytes = 128;   // one proxy row (dp <= 64 bf16) in a 128-byte swizzle slab

struct ScoreParams {
    int B, T, Hp, dp, nblk, npair, topk, RB, qb0, per_group;
    const __nv_bfloat16* qp;
    const int32_t* ptr2;
    const int32_t* off2;
    const int32_t* tok2;
    float* zsel;       // [entry][2]
    int32_t* jsel;     // [entry][2]
    uint32_t* status;
};

// One accumulator of 256 TMEM columns per CTA, so that two CTAs share an SM
// and one's epilogue overlaps the other's MMA.
__global__ void __launch_bounds__(kScThreads, 2)
proxy_grad_scores_kernel(const __grid_constant__ CUtensorMap tm_kp, ScoreParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int qe = 0;
    const RangeItem item = pair_item((int)blockIdx.x, p.nblk, p.npair, p.RB, p.qb0, p.per_group, p.ptr2, p.off2, &qe);
    const int pn = item.n, bg = item.bg, n0 = 2 * pn;
    const int nsub = n0 + 1 < qe ? 2 : 1;
    const int b = bg / p.Hp, g = bg % p.Hp;
    const int count = item.count;
    if (count <= 0) return;
    const uint32_t code0 = kStTimeoutBase + kKidProxy * 16 + 8;
    if ((smem_u32(smem) & 1023u) != 0u) {
        if (threadIdx.x == 0) atomicCAS(p.status, 0u, code0 + 7);
        return;
    }
    const int64_t ent0 = (int64_t)bg * p.T * p.topk + item.beg;   // first entry of the item
    const int32_t* toks = p.tok2 + ent0;
    const int nchunks = (count + 127) / 128;

    uint8_t* kp_tile = smem;                       // 256 keys x 128 B
    uint8_t* q_st = smem + 256 * kRowBytes;        // 2 stages of 128 queries x 128 B
    uint64_t* bars = (uint64_t*)(smem + 256 * kRowBytes + 2 * 128 * kRowBytes);
    uint64_t* kv_full = bars;
    uint64_t* q_full = bars + 1;     // [2]
    uint64_t* q_empty = q_full + 2;  // [2]
    uint64_t* a_full = q_empty + 2;  // MMA -> epilogue
    uint64_t* a_empty = a_full + 1;  // epilogue -> MMA
    uint64_t* fin = a_empty + 1;
    uint32_t* tmem_hold = (uint32_t*)(fin + 1);
    volatile uint32_t* abort_flag = tmem_hold + 1;
    const WaitCtx wc{p.status, abort_flag, MSA_WAIT_LIMIT_NS};

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&q_full[s], 128);
            mbar_init(&q_empty[s], 1);
        }
        mbar_init(a_full, 1);
        mbar_init(a_empty, 128);
        mbar_init(fin, 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 1) { tmem_alloc(tmem_hold, 256); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_hold;   // one accumulator of 256 columns

    if (warp == 0) {
        if (lane == 0) {   // the pair's 256 proxy keys, one box
            tma_prefetch_desc(&tm_kp);
            mbar_arrive_expect_tx(kv_full, 256 * kRowBytes);
            tma_load_4d(kp_tile, &tm_kp, kv_full, 0, g, n0 * 128, b);
            mbar_drain(kv_full, 0);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, 256, false, false);
            const int ksteps = (p.dp + 15) / 16;
            const uint32_t ka = smem_u32(kp_tile);
            bool ok = mbar_wait(kv_full, 0, wc, code0 + 0);
            for (int c = 0; ok && c < nchunks; ++c) {
                const int s = c & 1;
                const uint32_t use = (uint32_t)(c >> 1);
                if (!mbar_wait(&q_full[s], use & 1u, wc, code0 + 1)) break;
                if (c > 0 && !mbar_wait(a_empty, (uint32_t)(c - 1) & 1u, wc, code0 + 2)) break;
                tc_fence_after();
                const uint32_t qa = smem_u32(q_st + s * 128 * kRowBytes);
                for (int kk = 0; kk < ksteps; ++kk)
                    umma_ss(tmem, desc_kmajor(qa, 128, kk * 16), desc_kmajor(ka, 256, kk * 16), idesc,
                            kk > 0 ? 1u : 0u);
                umma_commit(&q_empty[s]);
                umma_commit(a_full);
            }
            umma_commit(fin);
            mbar_drain(fin, 0);
        }
    } else if (warp < 6) {
        // ---------------- proxy-query gather: 128 rows x 8 pieces of 16 B ----------------
        const int tid = threadIdx.x - 64;
        const int pieces = p.dp / 8;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const uint32_t use = (uint32_t)(c >> 1);
            if (use > 0 && !mbar_wait(&q_empty[s], (use - 1) & 1u, wc, code0 + 3)) break;
            const uint32_t qs = smem_u32(q_st + s * 128 * kRowBytes);
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int piece = it * 128 + tid, row = piece >> 3, ch = piece & 7;
                const int jj = c * 128 + row;
                const bool valid = jj < count && ch < pieces;
                const int i = jj < count ? (toks[jj] >> 2) : 0;
                const __nv_bfloat16* src = p.qp + (((int64_t)b * p.T + i) * p.Hp + g) * p.dp + (valid ? ch * 8 : 0);
                cp_async_16(qs + sw128_offset(row, ch, 0, 128), src, valid ? 16u : 0u);
            }
            cp_async_commit();
            cp_async_wait<0>();
            fence_proxy_async_smem();
            mbar_arrive(&q_full[s]);
        }
        cp_async_wait<0>();
    } else {
        // ---------------- epilogue: z and the argmax key of each selected block ----------------
        const int r = ((warp & 3) << 5) | lane;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
        for (int c = 0; c < nchunks; ++c) {
            const bool ok = mbar_wait(a_full, (uint32_t)c & 1u, wc, code0 + 4);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int jj = c * 128 + r;
            const int ent = jj < count ? toks[jj] : -1;
            const int i = ent >> 2, flags = ent >= 0 ? (ent & 3) : 0;
            for (int sb = 0; sb < nsub; ++sb) {
                const int cmax = !((flags >> sb) & 1) ? -1 : (((i >> 7) == n0 + sb) ? (i & 127) : 127);
                float best = -INFINITY;
                int arg = 0;
#pragma unroll
                for (int piece = 0; piece < 4; ++piece) {
                    uint32_t v[32];
                    tmem_ld32(tmem_addr(tmem, lane_base, (uint32_t)sb * 128u + piece * 32), v);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int col = piece * 32 + e;
                        const float x = __uint_as_float(v[e]);
                        if (col <= cmax && x > best) { best = x; arg = col; }   // strict: the lowest key on ties
                    }
                }
                if (cmax >= 0) {
                    p.zsel[(ent0 + jj) * 2 + sb] = best;
                    p.jsel[(ent0 + jj) * 2 + sb] = (n0 + sb) * 128 + arg;
                }
            }
            tc_fence_before();
            mbar_arrive(a_empty);
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// One CTA per (b, group, query tile); a warp walks its 32 rows one by one,
// its lanes over the row's selected blocks (up to 4 each), then over the
// proxy dims for dqp.
template <int G>
__global__ void __launch_bounds__(128, 4) proxy_grad_rows_kernel(
    const __nv_bfloat16* __restrict__ kp, const int32_t* __restrict__ idx, const int32_t* __restrict__ nsel,
    const int32_t* __restrict__ ptr2, const int32_t* __restrict__ off2, const float* __restrict__ bmass,
    const float* __restrict__ zsel, const int32_t* __restrict__ jsel, int T, int Hp, int dp, int topk, int nblk,
    int npair, int qb0, float* __restrict__ dz, float* __restrict__ dqp, float* __restrict__ loss)
{
    extern __shared__ uint32_t mask[];
    const int qb = qb0 + (int)blockIdx.x, bg = blockIdx.y, b = bg / Hp, g = bg % Hp;
    build_masks(mask, idx, nsel, T, topk, qb, bg);   // malformed entries: reported by the index build
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t* pp = ptr2 + (int64_t)bg * (npair + 1);
    const int32_t* offrow = off2 + ((int64_t)bg * nblk + qb) * npair;
    const int64_t ebase = (int64_t)bg * T * topk;
    for (int rr = 0; rr < 32; ++rr) {
        const int t = warp * 32 + rr, i = qb * 128 + t;
        if (i >= T) break;   // warp-uniform
        const int64_t srow = (int64_t)bg * T + i;
        int ns = nsel[srow];
        ns = ns < 0 ? 0 : (ns > topk ? topk : ns);
        // this lane's slots s = lane + 32 k: entry (e * 2 + sub) of each
        int64_t ek[4];
        bool vk[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int s = lane + 32 * k;
            const int n = s < ns ? idx[srow * topk + s] : -1;
            vk[k] = n >= 0 && n <= qb;
            ek[k] = 0;
            if (vk[k]) {
                const int pr = n >> 1;
                int rank = 0;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint32_t u = mask[(2 * pr) * 4 + w] | (2 * pr + 1 <= qb ? mask[(2 * pr + 1) * 4 + w] : 0u);
                    const int lo = t - 32 * w;
                    rank += lo >= 32 ? __popc(u) : (lo > 0 ? __popc(u & ((1u << lo) - 1u)) : 0);
                }
                ek[k] = (ebase + pp[pr] + offrow[pr] + rank) * 2 + (n & 1);
            }
        }
        // p: each head's weights normalised over the row's blocks, averaged over the heads
        float pk[4] = {0.f, 0.f, 0.f, 0.f};
        int heads = 0;
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
            float m[4], tot = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                m[k] = vk[k] ? bmass[ek[k] * G + hh] : 0.f;
                tot += m[k];
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
            if (tot > 0.f && tot <= 3.0e38f) {   // a head whose sums are not usable adds nothing
                ++heads;
#pragma unroll
                for (int k = 0; k < 4; ++k) pk[k] += m[k] / tot;
            }
        }
        const float invh = heads > 0 ? 1.f / (float)heads : 0.f;
        float zk[4], zmax = -INFINITY, psum = 0.f;
        int jk[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            pk[k] *= invh;
            zk[k] = vk[k] ? zsel[ek[k]] : -INFINITY;
            jk[k] = vk[k] ? jsel[ek[k]] : 0;
            zmax = fmaxf(zmax, zk[k]);
            psum += pk[k];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, off));
            psum += __shfl_xor_sync(0xffffffffu, psum, off);
        }
        float se = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) se += vk[k] ? expf(zk[k] - zmax) : 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) se += __shfl_xor_sync(0xffffffffu, se, off);
        const float lse_z = zmax + logf(se);
        float lsum = 0.f, dzk[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float lq = zk[k] - lse_z;
            dzk[k] = vk[k] ? expf(lq) * psum - pk[k] : 0.f;
            if (vk[k] && pk[k] > 0.f) lsum += pk[k] * (logf(pk[k]) - lq);
            if (vk[k]) dz[ek[k]] = dzk[k];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
        // dqp_i = sum over the row's blocks of dz kp_j*: lanes over dims
        const int d0 = 2 * lane;
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (32 * k >= ns) continue;   // warp-uniform
#pragma unroll 8
            for (int l = 0; l < 32; ++l) {
                const float dzs = __shfl_sync(0xffffffffu, dzk[k], l);
                const int js = __shfl_sync(0xffffffffu, jk[k], l);
                if (32 * k + l < ns && dzs != 0.f && d0 < dp) {
                    const __nv_bfloat162 kv =
                        *reinterpret_cast<const __nv_bfloat162*>(kp + (((int64_t)b * T + js) * Hp + g) * dp + d0);
                    const float2 f = __bfloat1622float2(kv);
                    a0 = fmaf(dzs, f.x, a0);
                    a1 = fmaf(dzs, f.y, a1);
                }
            }
        }
        if (d0 < dp) {
            float* out = dqp + (((int64_t)b * T + i) * Hp + g) * dp + d0;
            out[0] = a0;
            out[1] = a1;
        }
        if (lane == 0) loss[srow] = lsum;
    }
}

// dkp of the 256 keys of pair pn of one group, from the entries of the pair
// list: up to kKeySplit CTAs per pair, each over its share of the entries
// with shared-memory fp32 accumulators [256][dp + 1], added into dkp at the
// end (the pair holding block 0 is selected by every row: at 1M tokens one
// CTA would walk a million entries).  A warp takes
// four entries at a time, its lanes over the proxy dims (two each): the
// argmax keys of many rows coincide, so lanes must not add to the same key
// row at once; the four entries' loads are all in flight together.
constexpr int kKeyMinChunk = 2048;   // entries: fewer go to one CTA
constexpr int kKeySplit = 16;        // at most this many CTAs per pair

__global__ void __launch_bounds__(256) proxy_grad_keys_kernel(
    const __nv_bfloat16* __restrict__ qp, const int32_t* __restrict__ ptr2, const int32_t* __restrict__ tok2,
    const int32_t* __restrict__ jsel, const float* __restrict__ dz, int T, int Hp, int dp, int topk, int npair,
    float* __restrict__ dkp)
{
    extern __shared__ float acc[];   // [256][dp + 1]
    const int ld = dp + 1;
    const int pn = blockIdx.x, bg = blockIdx.y, b = bg / Hp, g = bg % Hp;
    // this CTA's share of the pair's entry list: gridDim.z equal parts of at
    // least kKeyMinChunk entries (a heavily shared pair, such as the one
    // holding block 0, is spread over several CTAs instead of one)
    const int p0 = ptr2[(int64_t)bg * (npair + 1) + pn], p1 = ptr2[(int64_t)bg * (npair + 1) + pn + 1];
    const int cs = max(kKeyMinChunk, (p1 - p0 + (int)gridDim.z - 1) / (int)gridDim.z);
    const int e0 = p0 + (int)blockIdx.z * cs;
    if (e0 >= p1) return;   // CTA-uniform
    const int e1 = min(p1, e0 + cs);
    for (int x = threadIdx.x; x < 256 * ld; x += blockDim.x) acc[x] = 0.f;
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d0 = 2 * lane;
    const int64_t ebase = (int64_t)bg * T * topk;
    constexpr int kE = 4;   // entries per warp step
    for (int base = e0 + warp * kE; base < e1; base += 8 * kE) {
        // lane l < 2 kE loads (entry l / 2, block l % 2): its flags, weight and key
        const int le = base + (lane >> 1), lsb = lane & 1;
        int lent = 0, lkey = -1;
        float lw = 0.f;
        if (lane < 2 * kE && le < e1) {
            // the three loads are independent: the weight and key slots exist for
            // every entry and are used only when the entry selected the block
            const int64_t x = (ebase + le) * 2 + lsb;
            lent = tok2[ebase + le];
            const float w = dz[x];
            const int key = jsel[x];
            if ((lent >> lsb) & 1) {
                lw = w;
                lkey = key - 256 * pn;   // 0 .. 255
            }
        }
        float2 q[kE];
#pragma unroll
        for (int u = 0; u < kE; ++u) {
            const int ent = __shfl_sync(0xffffffffu, lent, 2 * u);
            q[u] = make_float2(0.f, 0.f);
            if (base + u < e1 && d0 < dp)
                q[u] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(
                    qp + (((int64_t)b * T + (ent >> 2)) * Hp + g) * dp + d0));
        }
#pragma unroll
        for (int u = 0; u < 2 * kE; ++u) {
            const float w = __shfl_sync(0xffffffffu, lw, u);
            const int key = __shfl_sync(0xffffffffu, lkey, u);
            if (w != 0.f && key >= 0 && key < 256 && d0 < dp) {
                atomicAdd(acc + key * ld + d0, w * q[u >> 1].x);
                atomicAdd(acc + key * ld + d0 + 1, w * q[u >> 1].y);
            }
        }
    }
    __syncthreads();
    // add the partial sums into dkp (zeroed before the launch); most keys of
    // a pair are nobody's argmax and are skipped
    for (int x = threadIdx.x; x < 256 * dp; x += blockDim.x) {
        const int k = x / dp, d = x % dp, j = 256 * pn + k;
        const float v = acc[k * ld + d];
        if (j < T && v != 0.f) atomicAdd(dkp + (((int64_t)b * T + j) * Hp + g) * dp + d, v);
    }
}

template <int G>
cudaError_t launch_rows(const Problem& pr, const void* kp, const int32_t* idx, const int32_t* nsel,
                        const int32_t* ptr2, const int32_t* off2, const float* bmass, const float* zsel,
                        const int32_t* jsel, float* dz, float* dqp, float* loss, cudaStream_t st)
{
    const size_t mask_bytes = (size_t)pr.nblk * 16;
    if (mask_bytes > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(proxy_grad_rows_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)mask_bytes);
        if (e != cudaSuccess) return e;
    }
    proxy_grad_rows_kernel<G><<<dim3((unsigned)(pr.nblk - pr.qb0), (unsigned)(pr.B * pr.Hp)), 128, mask_bytes, st>>>(
        (const __nv_bfloat16*)kp, idx, nsel, ptr2, off2, bmass, zsel, jsel, pr.T, pr.Hp, pr.dp, pr.topk, pr.nblk,
        pair_count(pr.nblk), pr.qb0, dz, dqp, loss);
    count_launches(1);
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_proxy_bwd(const Problem& pr, const CUtensorMap& tm_kp, const void* qp, const void* kp,
                             const int32_t* idx, const int32_t* nsel, float* dqp, float* dkp, float* loss,
                             void* ws, const WsLayout& L, cudaStream_t st)
{
    uint8_t* w = (uint8_t*)ws;
    const int32_t* ptr2 = (const int32_t*)(w + L.ptr2);
    const int32_t* off2 = (const int32_t*)(w + L.cnt2);
    const int32_t* tok2 = (const int32_t*)(w + L.tok2);
    float* zsel = (float*)(w + L.zsel);
    int32_t* jsel = (int32_t*)(w + L.jsel);
    float* dz = (float*)(w + L.dz);
    const float* bmass = (const float*)(w + L.bmass);
    const int npair = pair_count(pr.nblk);

    ScoreParams sp;
    sp.B = pr.B; sp.T = pr.T; sp.Hp = pr.Hp; sp.dp = pr.dp; sp.nblk = pr.nblk; sp.npair = npair; sp.topk = pr.topk;
    sp.RB = range_blocks(pr);
    sp.qb0 = pr.qb0;
    sp.per_group = pair_items_per_group(pr.nblk, sp.RB, pr.qb0);
    sp.qp = (const __nv_bfloat16*)qp;
    sp.ptr2 = ptr2; sp.off2 = off2; sp.tok2 = tok2;
    sp.zsel = zsel; sp.jsel = jsel;
    sp.status = (uint32_t*)(w + L.status);
    const size_t smem = 1024 + 256 * kRowBytes + 2 * 128 * kRowBytes + 16 * 8;
    cudaError_t e = cudaFuncSetAttribute(proxy_grad_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    proxy_grad_scores_kernel<<<(unsigned)(sp.per_group * pr.B * pr.Hp), kScThreads, smem, st>>>(tm_kp, sp);
    count_launches(1);

    switch (pr.G) {
    case 1: e = launch_rows<1>(pr, kp, idx, nsel, ptr2, off2, bmass, zsel, jsel, dz, dqp, loss, st); break;
    case 2: e = launch_rows<2>(pr, kp, idx, nsel, ptr2, off2, bmass, zsel, jsel, dz, dqp, loss, st); break;
    case 4: e = launch_rows<4>(pr, kp, idx, nsel, ptr2, off2, bmass, zsel, jsel, dz, dqp, loss, st); break;
    case 8: e = launch_rows<8>(pr, kp, idx, nsel, ptr2, off2, bmass, zsel, jsel, dz, dqp, loss, st); break;
    default: e = launch_rows<16>(pr, kp, idx, nsel, ptr2, off2, bmass, zsel, jsel, dz, dqp, loss, st); break;
    }
    if (e != cudaSuccess) return e;

    const size_t kbytes = (size_t)256 * (pr.dp + 1) * 4;
    if ((e = cudaFuncSetAttribute(proxy_grad_keys_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kbytes)) !=
        cudaSuccess)
        return e;
    if ((e = cudaMemsetAsync(dkp, 0, sizeof(float) * (size_t)pr.B * pr.T * pr.Hp * pr.dp, st)) != cudaSuccess)
        return e;
    proxy_grad_keys_kernel<<<dim3((unsigned)npair, (unsigned)(pr.B * pr.Hp), (unsigned)kKeySplit), 256, kbytes, st>>>(
        (const __nv_bfloat16*)qp, ptr2, tok2, jsel, dz, pr.T, pr.Hp, pr.dp, pr.topk, npair, dkp);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace msa
