// Index Branch: proxy score GEMM + causal block max-pool + top-k selection.
//
// Method (page "Flash-MSA: Open-Source Sparse Attention Kernels Debut",
// section "How MSA works"): each GQA group has one proxy head; its scores
// over all causal (query, key) pairs are max-pooled into 128-key blocks and
// each query picks the blocks it will read; the picked ids are cached.
//
// One CTA owns one (batch, group, 128-query tile qb).  The proxy query tile
// stays in shared memory; proxy key tiles n = 0 .. qb-1 stream in through a
// 4-stage TMA ring; one thread issues tcgen05 MMAs (M=128 queries, N=128
// keys, K=dp) into a double-buffered TMEM accumulator; four epilogue warps
// (one TMEM lane = one query row each) reduce each 128-column tile to its
// max and feed it into the row's selection heap in shared memory.  The
// diagonal tile is needed only for the optional pooled-score output: the own
// block is always selected, so selection only ranks blocks 0 .. qb-1, which
// every query of the tile sees in full (no causal mask there).
//
// Selection order: higher pooled score first, equal scores to the lower
// block id.  Tiles arrive in ascending n, so a later tile displaces the heap
// root (the current worst) only with a strictly greater score.
#include <math.h>

#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kStages = 4;
constexpr int kThreads = 192;             // warp 0: TMA, warp 1: MMA, warps 2-5: epilogue
constexpr uint32_t kTileBytes = 128 * 128; // 128 rows x 64 bf16 (one 128-byte swizzle slab)
constexpr uint32_t kTmemCols = 256;        // two 128-column fp32 accumulators

struct Params {
    int B, T, Hp, dp, nblk, topk;
    int32_t* idx;
    int32_t* nsel;
    float* pooled;     // optional
    uint32_t* status;
};

MSA_DEV bool worse(float sa, int ia, float sb, int ib)
{
    return sa < sb || (sa == sb && ia > ib);
}

// Column r of the [slot][128] heap arrays: a binary heap whose root is the
// worst kept candidate.
MSA_DEV void sift_down(float* hs, int* hi, int k1, int r, int x)
{
    const float sx = hs[x * 128 + r];
    const int ix = hi[x * 128 + r];
    for (;;) {
        const int l = 2 * x + 1;
        if (l >= k1) break;
        int w = l;
        float sw = hs[l * 128 + r];
        int iw = hi[l * 128 + r];
        if (l + 1 < k1) {
            const float s2 = hs[(l + 1) * 128 + r];
            const int i2 = hi[(l + 1) * 128 + r];
            if (worse(s2, i2, sw, iw)) { w = l + 1; sw = s2; iw = i2; }
        }
        if (!worse(sw, iw, sx, ix)) break;
        hs[x * 128 + r] = sw;
        hi[x * 128 + r] = iw;
        x = w;
    }
    hs[x * 128 + r] = sx;
    hi[x * 128 + r] = ix;
}

__global__ void __launch_bounds__(kThreads, 1)
proxy_select_kernel(const __grid_constant__ CUtensorMap tm_qp, const __grid_constant__ CUtensorMap tm_kp,
                    Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int BH = p.B * p.Hp;
    const int qb = p.nblk - 1 - (int)(blockIdx.x / BH);   // heaviest tiles first
    const int bg = (int)(blockIdx.x % BH);
    const int b = bg / p.Hp, g = bg % p.Hp;
    const int k1 = p.topk - 1;                             // slots besides the own block
    const bool dbg = p.pooled != nullptr;
    const bool take_all = qb + 1 <= p.topk;                // every eligible block kept
    const bool need_heap = !take_all && k1 > 0;
    const int ntiles = dbg ? qb + 1 : (need_heap ? qb : 0);

    // epilogue row of this thread (warps 2..5 own TMEM lane quarters 2,3,0,1)
    const int r = ((warp & 3) << 5) | lane;
    const int i = qb * 128 + r;
    const bool row_ok = (warp >= 2) && (i < p.T);

    uint8_t* qp_tile = smem;
    uint8_t* kp_tiles = smem + kTileBytes;
    float* heap_s = (float*)(smem + kTileBytes * (1 + kStages));
    int* heap_i = (int*)(heap_s + (size_t)(k1 > 0 ? k1 : 0) * 128);
    uint64_t* bars = (uint64_t*)(heap_i + (size_t)(k1 > 0 ? k1 : 0) * 128);
    uint64_t* full = bars;                 // [kStages] TMA -> MMA
    uint64_t* empty = bars + kStages;      // [kStages] MMA -> TMA
    uint64_t* acc_full = bars + 2 * kStages;   // [2] MMA -> epilogue
    uint64_t* acc_empty = acc_full + 2;        // [2] epilogue -> MMA
    uint64_t* qp_full = acc_empty + 2;
    uint64_t* fin = qp_full + 1;               // MMA teardown drain
    uint32_t* tmem_hold = (uint32_t*)(fin + 1);
    volatile uint32_t* abort_flag = tmem_hold + 1;
    const WaitCtx wc{p.status, abort_flag, MSA_WAIT_LIMIT_NS};
    const uint32_t code0 = kStTimeoutBase + kKidProxy * 16;

    if (ntiles == 0) {
        // Nothing to rank: the query keeps blocks 0..qb (or only qb when topk == 1).
        if (row_ok) {
            int32_t* out = p.idx + ((int64_t)bg * p.T + i) * p.topk;
            int c = 0;
            if (take_all) {
                for (int n = 0; n <= qb; ++n) out[c++] = n;
            } else {
                out[c++] = qb;
            }
            p.nsel[(int64_t)bg * p.T + i] = c;
            for (int s = c; s < p.topk; ++s) out[s] = -1;
        }
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int s = 0; s < 2; ++s) { mbar_init(&acc_full[s], 1); mbar_init(&acc_empty[s], 128); }
        mbar_init(qp_full, 1);
        mbar_init(fin, 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 1) { tmem_alloc(tmem_hold, kTmemCols); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_hold;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_qp);
            tma_prefetch_desc(&tm_kp);
            mbar_arrive_expect_tx(qp_full, kTileBytes);
            tma_load_4d(qp_tile, &tm_qp, qp_full, 0, g, qb * 128, b);
            int n = 0;
            for (; n < ntiles; ++n) {
                const int s = n % kStages;
                const uint32_t use = (uint32_t)(n / kStages);
                if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1u, wc, code0 + 0)) break;
                mbar_arrive_expect_tx(&full[s], kTileBytes);
                tma_load_4d(kp_tiles + s * kTileBytes, &tm_kp, &full[s], 0, g, n * 128, b);
            }
            if (*abort_flag) {   // let copies still in flight land before the CTA exits
                mbar_drain(qp_full, 0);
                for (int m = (n > kStages ? n - kStages : 0); m < n; ++m)
                    mbar_drain(&full[m % kStages], (uint32_t)(m / kStages) & 1u);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, 128, false, false);
            const int ksteps = (p.dp + 15) / 16;
            const uint32_t a0 = smem_u32(qp_tile);
            bool ok = mbar_wait(qp_full, 0, wc, code0 + 1);
            for (int n = 0; ok && n < ntiles; ++n) {
                const int s = n % kStages;
                const uint32_t use = (uint32_t)(n / kStages);
                const int buf = n & 1;
                const uint32_t ause = (uint32_t)(n >> 1);
                if (!mbar_wait(&full[s], use & 1u, wc, code0 + 2)) break;
                if (ause > 0 && !mbar_wait(&acc_empty[buf], (ause - 1) & 1u, wc, code0 + 3)) break;
                tc_fence_after();
                const uint32_t b0 = smem_u32(kp_tiles + s * kTileBytes);
                for (int kk = 0; kk < ksteps; ++kk)
                    umma_ss(tmem + buf * 128, desc_kmajor(a0, 128, kk * 16),
                            desc_kmajor(b0, 128, kk * 16), idesc, kk > 0 ? 1u : 0u);
                umma_commit(&empty[s]);
                umma_commit(&acc_full[buf]);
            }
            umma_commit(fin);     // every MMA issued above has finished once this fires
            mbar_drain(fin, 0);
        }
    } else {
        // ---------------- epilogue: pool + select ----------------
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
        int cnt = 0;
        for (int n = 0; n < ntiles; ++n) {
            const int buf = n & 1;
            const uint32_t use = (uint32_t)(n >> 1);
            bool ok = mbar_wait(&acc_full[buf], use & 1u, wc, code0 + 4);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t ta = tmem_addr(tmem, lane_base, (uint32_t)buf * 128u);
            const bool diag = (n == qb);
            float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t v[64];
                tmem_ld32(ta + half * 64, v);
                tmem_ld32(ta + half * 64 + 32, v + 32);
                tmem_ld_wait();
                if (diag) {
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (half * 64 + c > r) v[c] = __float_as_uint(-INFINITY);
                }
#pragma unroll
                for (int c = 0; c < 64; c += 8) {
                    m0 = fmax3(m0, __uint_as_float(v[c + 0]), __uint_as_float(v[c + 1]));
                    m1 = fmax3(m1, __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
                    m2 = fmax3(m2, __uint_as_float(v[c + 4]), __uint_as_float(v[c + 5]));
                    m3 = fmax3(m3, __uint_as_float(v[c + 6]), __uint_as_float(v[c + 7]));
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[buf]);
            const float mx = fmaxf(fmax3(m0, m1, m2), m3);
            if (dbg && row_ok) p.pooled[((int64_t)bg * p.T + i) * p.nblk + n] = mx;
            if (need_heap && !diag) {
                if (cnt < k1) {
                    heap_s[cnt * 128 + r] = mx;
                    heap_i[cnt * 128 + r] = n;
                    if (++cnt == k1)
                        for (int x = k1 / 2 - 1; x >= 0; --x) sift_down(heap_s, heap_i, k1, r, x);
                } else if (mx > heap_s[r]) {
                    heap_s[r] = mx;
                    heap_i[r] = n;
                    sift_down(heap_s, heap_i, k1, r, 0);
                }
            }
        }
        if (row_ok && !*abort_flag) {
            int32_t* out = p.idx + ((int64_t)bg * p.T + i) * p.topk;
            int c = 0;
            if (take_all) {
                for (int n = 0; n <= qb; ++n) out[c++] = n;
            } else if (k1 == 0) {
                out[c++] = qb;
            } else {
                // ascending block ids: insertion sort of the heap column
                for (int a = 1; a < k1; ++a) {
                    const int key = heap_i[a * 128 + r];
                    int x = a - 1;
                    while (x >= 0 && heap_i[x * 128 + r] > key) {
                        heap_i[(x + 1) * 128 + r] = heap_i[x * 128 + r];
                        --x;
                    }
                    heap_i[(x + 1) * 128 + r] = key;
                }
                for (int a = 0; a < k1; ++a) out[c++] = heap_i[a * 128 + r];
                out[c++] = qb;
            }
            p.nsel[(int64_t)bg * p.T + i] = c;
            for (int s = c; s < p.topk; ++s) out[s] = -1;
            if (dbg)
                for (int n = qb + 1; n < p.nblk; ++n)
                    p.pooled[((int64_t)bg * p.T + i) * p.nblk + n] = -INFINITY;
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_proxy_select(const Problem& pr, const CUtensorMap& tm_qp, const CUtensorMap& tm_kp,
                                int32_t* idx, int32_t* nsel, float* pooled, uint32_t* status,
                                cudaStream_t st)
{
    Params p{pr.B, pr.T, pr.Hp, pr.dp, pr.nblk, pr.topk, idx, nsel, pooled, status};
    const size_t k1 = (size_t)(pr.topk - 1);
    const size_t smem = 1024 + (size_t)kTileBytes * (1 + kStages) + k1 * 128 * 8 + 16 * 8 + 16;
    cudaError_t e = cudaFuncSetAttribute(proxy_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(pr.nblk * pr.B * pr.Hp);
    trace_begin(kTraceProxy, st);
    proxy_select_kernel<<<grid, kThreads, smem, st>>>(tm_qp, tm_kp, p);
    trace_end(kTraceProxy, st);
    return cudaGetLastError();
}

}  // namespace msa
