// Index Branch: proxy score GEMM + causal block max-pool + top-k selection.
//
// Method (page "Flash-MSA: Open-Source Sparse Attention Kernels Debut",
// section "How MSA works"): each GQA group has one proxy head; its scores
// over all causal (query, key) pairs are max-pooled into 128-key blocks and
// each query picks the blocks it will read; the picked ids are cached.
//
// One CTA owns one (batch, group, 128-query tile qb).  The proxy query tile
// stays in shared memory; proxy key tiles n = 0 .. qb-1 stream in through a
// TMA ring two key blocks at a time; one thread issues tcgen05 MMAs (M=128
// queries, N=256 keys, K=dp; one N=128 chain per block measured slower: twice
// the MMAs and hand-offs for the same work) into two TMEM accumulators; eight
// pooling warps (one TMEM lane = one query row each; two warps per lane
// quarter, one per key block of the 256-key MMA) reduce each 128-column
// block to its max, free the
// accumulator and pass the maxima through a shared-memory ring to four
// selection warps, which own the rows' selection state.  Pooling and
// selection thus overlap, and the accumulator is handed back to the MMA as
// soon as it has been read.  The diagonal tile is needed only for the optional
// pooled-score output: the own block is always selected, so selection only
// ranks blocks 0 .. qb-1, which every query of the tile sees in full.
//
// Selection state per row (shared memory, [slot][row] so a warp touches 32
// distinct banks): a 4-ary heap of the best topk-1 (score, id) pairs whose
// root is the worst kept pair, and a small pending list.  At the end each
// selection thread sorts its own row's kept ids with a bitonic network in
// registers (topk <= 64; larger topk: one row at a time across the warp's
// lanes).  Key tiles are
// scanned nearest-first (descending block id): under causal locality the
// best blocks tend to be the recent ones, so after the first few tiles a
// new tile rarely beats the heap root.  A new tile has a lower id than every
// kept pair, so it displaces the root when its score is greater or equal; a
// tile beating the root (kept in a register) is appended to the pending
// list, and the warp merges pending lists into the heaps only when one of
// its rows fills its list.  Order: higher score first, equal scores to the
// lower block id.
//
// CTAs run group by group, heaviest query tiles first, so the proxy keys of
// one group stay in L2 while its tiles are processed.
#include <math.h>

#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kThreads = 448;             // warp 0: TMA, 1: MMA, 2-9: pooling, 10-13: selection
constexpr uint32_t kTileBytes = 128 * 128; // 128 rows x 64 bf16 (one 128-byte swizzle slab)
constexpr int kPend = 10;                  // pending slots per row (merge once one row holds 6)
constexpr int kNacc = 2;                   // TMEM accumulators (256 columns each)

struct Params {
    int B, T, Hp, dp, nblk, topk;
    int qb0;                // first query tile computed (earlier tiles are skipped)
    int window, dilation;   // forced blocks: qb, qb - dilation, ... (window of them)
    int32_t* idx;
    int32_t* nsel;
    float* pooled;     // optional
    uint32_t* status;
};

// A candidate is (score bits, block id) in one 64-bit word.
MSA_DEV uint2 cand(float s, int n) { return make_uint2(__float_as_uint(s), (uint32_t)n); }

MSA_DEV bool worse(uint2 a, uint2 b)
{
    const float sa = __uint_as_float(a.x), sb = __uint_as_float(b.x);
    return sa < sb || (sa == sb && (int)a.y > (int)b.y);
}

// Column r of the [slot][128] heap array: a 4-ary heap whose root is the
// worst kept candidate (children of x are 4x+1 .. 4x+4: half the depth of a
// binary heap; the four children are loaded together, indices past the end
// repeating the last child).
MSA_DEV void sift_down(uint2* h, int k1, int r, int x)
{
    const uint2 ex = h[x * 128 + r];
    const int last = k1 - 1;
    for (;;) {
        const int c0 = 4 * x + 1;
        if (c0 > last) break;
        const int c1 = min(c0 + 1, last), c2 = min(c0 + 2, last), c3 = min(c0 + 3, last);
        const uint2 e0 = h[c0 * 128 + r], e1 = h[c1 * 128 + r], e2 = h[c2 * 128 + r], e3 = h[c3 * 128 + r];
        int w = c0;
        uint2 ew = e0;
        if (worse(e1, ew)) { w = c1; ew = e1; }
        if (worse(e2, ew)) { w = c2; ew = e2; }
        if (worse(e3, ew)) { w = c3; ew = e3; }
        if (!worse(ew, ex)) break;
        h[x * 128 + r] = ew;
        x = w;
    }
    h[x * 128 + r] = ex;
}

// Ascending sort of the 32*V ints a warp holds V per lane (element
// V*lane + w in v[w]) by a bitonic network.
template <int V>
MSA_DEV void warp_sort(int (&v)[V])
{
    const int lane = (int)(threadIdx.x & 31u);
#pragma unroll
    for (int k = 2; k <= 32 * V; k <<= 1) {
#pragma unroll
        for (int s = k >> 1; s >= 1; s >>= 1) {
            if (s < V) {   // partner in the same lane
#pragma unroll
                for (int w = 0; w < V; ++w) {
                    const int wp = w ^ s;
                    if (wp > w) {
                        const bool up = ((V * lane + w) & k) == 0;
                        const int a = v[w], b = v[wp];
                        v[w] = up ? min(a, b) : max(a, b);
                        v[wp] = up ? max(a, b) : min(a, b);
                    }
                }
            } else {
                const int ls = s / V;   // partner lane distance
#pragma unroll
                for (int w = 0; w < V; ++w) {
                    const int j = V * lane + w;
                    const int other = __shfl_xor_sync(0xffffffffu, v[w], ls);
                    const bool up = (j & k) == 0, lower = (j & s) == 0;
                    v[w] = (up == lower) ? min(v[w], other) : max(v[w], other);
                }
            }
        }
    }
}

// The warp's 32 rows (TMEM lane quarter q): ascending output of each row's
// k1 kept ids and the topk - k1 forced blocks qb, qb - dil, ...; one row at a
// time, V ids per lane.
template <int V>
MSA_DEV void write_selection(const uint2* heap, int k1, int topk, int dil, int q, int qb, int T, int64_t row0,
                             int32_t* idx, int32_t* nsel)
{
    const int lane = (int)(threadIdx.x & 31u);
    for (int rr = 0; rr < 32; ++rr) {
        const int row = q * 32 + rr;
        int v[V];
#pragma unroll
        for (int w = 0; w < V; ++w) {
            const int slot = V * lane + w;
            v[w] = slot < k1 ? (int)heap[slot * 128 + row].y
                             : (slot < topk ? qb - (slot - k1) * dil : 0x7fffffff);
        }
        warp_sort<V>(v);
        const int i = qb * 128 + row;
        if (i < T) {
            int32_t* out = idx + (row0 + row) * topk;
#pragma unroll
            for (int w = 0; w < V; ++w) {
                const int slot = V * lane + w;
                if (slot < topk) out[slot] = v[w];
            }
            if (lane == 0) nsel[row0 + row] = topk;
        }
    }
}

// Ascending sort of N ints held by one thread (bitonic network, fully
// unrolled: every index is a compile-time constant, so v stays in registers).
template <int N>
MSA_DEV void thread_sort(int (&v)[N])
{
#pragma unroll
    for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const int a = v[i], b = v[l];
                    const bool up = (i & k) == 0;
                    v[i] = up ? min(a, b) : max(a, b);
                    v[l] = up ? max(a, b) : min(a, b);
                }
            }
        }
    }
}

// The warp's 32 rows (TMEM lane quarter q), topk <= N: every thread sorts
// its own row's k1 kept ids and the topk - k1 forced blocks in registers (all
// 32 rows at once, no shuffles), parks the result in shared memory ([row][N+1]
// ints: the odd row stride keeps both access patterns free of bank
// conflicts) and the warp writes the rows out coalesced.
template <int N>
MSA_DEV void write_selection_rows(const uint2* heap, int k1, int topk, int dil, int q, int qb, int T, int64_t row0,
                                  int32_t* idx, int32_t* nsel, int32_t* stg)
{
    const int lane = (int)(threadIdx.x & 31u);
    const int row = q * 32 + lane;
    int v[N];
#pragma unroll
    for (int s = 0; s < N; ++s)
        v[s] = s < k1 ? (int)heap[s * 128 + row].y : (s < topk ? qb - (s - k1) * dil : 0x7fffffff);
    thread_sort<N>(v);
#pragma unroll
    for (int s = 0; s < N; ++s) stg[row * (N + 1) + s] = v[s];
    __syncwarp();
    for (int rr = 0; rr < 32; ++rr) {
        const int r2 = q * 32 + rr;
        if (qb * 128 + r2 < T) {   // warp-uniform
            int32_t* out = idx + (row0 + r2) * topk;
            for (int s = lane; s < topk; s += 32) out[s] = stg[r2 * (N + 1) + s];
            if (lane == 0) nsel[row0 + r2] = topk;
        }
    }
}

// Output of a row that ranks nothing: every eligible block (take_all), or the
// nf forced blocks qb - (nf-1) dil, ..., qb.
MSA_DEV void write_unranked(int32_t* out, int32_t* nsel_out, bool take_all, int qb, int nf, int dil, int topk)
{
    int c = 0;
    if (take_all) {
        for (int n = 0; n <= qb; ++n) out[c++] = n;
    } else {
        for (int m = nf - 1; m >= 0; --m) out[c++] = qb - m * dil;
    }
    *nsel_out = c;
    for (int s = c; s < topk; ++s) out[s] = -1;
}

// NSTAGE stages of 256 proxy keys (two key blocks) each; two TMEM
// accumulators of 256 columns (all of TMEM: one CTA per SM); RING pairs of
// block maxima between the pooling and the selection warps.  WINDOW: a forced
// pattern beyond the own block is in use (a separate instance keeps the
// plain selection's inner loop unchanged).
template <int NSTAGE, int RING, bool WINDOW>
__global__ void __launch_bounds__(kThreads, 1)
proxy_select_kernel(const __grid_constant__ CUtensorMap tm_qp, const __grid_constant__ CUtensorMap tm_kp,
                    Params p)
{
    constexpr int NACC = kNacc;
    constexpr uint32_t kTmemCols = 512;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // group by group, heaviest (largest qb) tiles first within a group; only
    // the tiles qb0 .. nblk-1 are launched
    const int nq = p.nblk - p.qb0;
    const int bg = (int)(blockIdx.x / nq);
    const int qb = p.nblk - 1 - (int)(blockIdx.x % nq);
    const int b = bg / p.Hp, g = bg % p.Hp;
    const int nf = WINDOW ? min(p.window, qb / p.dilation + 1) : 1;   // forced blocks that exist
    const int k1 = p.topk - nf;                            // slots ranked by pooled score
    const bool dbg = p.pooled != nullptr;
    const bool take_all = qb + 1 <= p.topk;                // every eligible block kept
    const bool need_heap = !take_all && k1 > 0;
    const int ntiles = dbg ? qb + 1 : (need_heap ? qb : 0);
    const int npairs = (ntiles + 1) / 2;
    // pair k holds key blocks hi = ntiles-1-2k (nearest first) and lo = hi-1
    // (lo = -1 past the first block: that half is zero-filled and ignored)

    // row of this thread: a pooling warp reads TMEM lane quarter warp & 3;
    // selection warp 10 + q owns rows 32q .. 32q + 31
    const bool sel_warp = warp >= 10;
    const int r = sel_warp ? ((warp - 10) << 5) | lane : ((warp & 3) << 5) | lane;
    const int i = qb * 128 + r;
    const bool row_ok = sel_warp && (i < p.T);

    const int hk = k1 > 0 ? k1 : 0;
    uint8_t* qp_tile = smem;
    uint8_t* kp_tiles = smem + kTileBytes;
    uint2* heap = (uint2*)(smem + kTileBytes * (1 + 2 * NSTAGE));   // [topk-1][128]
    uint2* pend = heap + (size_t)hk * 128;                             // [kPend][128]
    constexpr int ring = RING;
    float* pm = (float*)(pend + kPend * 128);    // [ring][2][128]: block maxima (lo, hi) of a pair
    uint64_t* bars = (uint64_t*)(pm + ring * 2 * 128);
    uint64_t* full = bars;                     // [NSTAGE] TMA -> MMA
    uint64_t* empty = bars + NSTAGE;           // [NSTAGE] MMA -> TMA
    uint64_t* acc_full = bars + 2 * NSTAGE;    // [NACC] MMA -> epilogue
    uint64_t* acc_empty = acc_full + NACC;     // [NACC] epilogue -> MMA
    uint64_t* pm_full = acc_empty + NACC;      // [ring] pooling -> selection
    uint64_t* pm_empty = pm_full + ring;       // [ring] selection -> pooling
    uint64_t* qp_full = pm_empty + ring;
    uint64_t* fin = qp_full + 1;               // MMA teardown drain
    uint32_t* tmem_hold = (uint32_t*)(fin + 1);
    volatile uint32_t* abort_flag = tmem_hold + 1;
    const WaitCtx wc{p.status, abort_flag, MSA_WAIT_LIMIT_NS};
    const uint32_t code0 = kStTimeoutBase + kKidProxy * 16;

    if (ntiles == 0) {
        // Nothing to rank: every eligible block, or only the forced ones.
        if (row_ok)
            write_unranked(p.idx + ((int64_t)bg * p.T + i) * p.topk, p.nsel + (int64_t)bg * p.T + i, take_all, qb,
                           nf, p.dilation, p.topk);
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int s = 0; s < NACC; ++s) { mbar_init(&acc_full[s], 1); mbar_init(&acc_empty[s], 256); }
        for (int s = 0; s < ring; ++s) { mbar_init(&pm_full[s], 256); mbar_init(&pm_empty[s], 128); }
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
        // ---------------- TMA producer: one 256-key box per pair ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_qp);
            tma_prefetch_desc(&tm_kp);
            mbar_arrive_expect_tx(qp_full, kTileBytes);
            tma_load_4d(qp_tile, &tm_qp, qp_full, 0, g, qb * 128, b);
            int k = 0;
            for (; k < npairs; ++k) {
                const int s = k % NSTAGE;
                const uint32_t use = (uint32_t)(k / NSTAGE);
                if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1u, wc, code0 + 0)) break;
                const int lo = ntiles - 2 - 2 * k;   // may be -1: rows before 0 read as zeros
                mbar_arrive_expect_tx(&full[s], 2 * kTileBytes);
                tma_load_4d(kp_tiles + s * 2 * kTileBytes, &tm_kp, &full[s], 0, g, lo * 128, b);
            }
            if (*abort_flag) {   // let copies still in flight land before the CTA exits
                mbar_drain(qp_full, 0);
                for (int m = (k > NSTAGE ? k - NSTAGE : 0); m < k; ++m)
                    mbar_drain(&full[m % NSTAGE], (uint32_t)(m / NSTAGE) & 1u);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: M = 128 queries, N = 256 keys ----------------
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, 256, false, false);
            const int ksteps = (p.dp + 15) / 16;
            const uint32_t a0 = smem_u32(qp_tile);
            bool ok = mbar_wait(qp_full, 0, wc, code0 + 1);
            for (int k = 0; ok && k < npairs; ++k) {
                const int s = k % NSTAGE;
                const uint32_t use = (uint32_t)(k / NSTAGE);
                const int buf = k % NACC;
                const uint32_t ause = (uint32_t)(k / NACC);
                if (!mbar_wait(&full[s], use & 1u, wc, code0 + 2)) break;
                if (ause > 0 && !mbar_wait(&acc_empty[buf], (ause - 1) & 1u, wc, code0 + 3)) break;
                tc_fence_after();
                const uint32_t b0 = smem_u32(kp_tiles + s * 2 * kTileBytes);
                for (int kk = 0; kk < ksteps; ++kk)
                    umma_ss(tmem + buf * 256, desc_kmajor(a0, 128, kk * 16),
                            desc_kmajor(b0, 256, kk * 16), idesc, kk > 0 ? 1u : 0u);
                umma_commit(&empty[s]);
                umma_commit(&acc_full[buf]);
            }
            umma_commit(fin);     // every MMA issued above has finished once this fires
            mbar_drain(fin, 0);
        }
    } else if (!sel_warp) {
        // ---------------- pooling: one 128-key block per warp and pair ----------------
        // warps 2-5 reduce the nearer block of each pair (accumulator columns
        // 128..255), warps 6-9 the farther one (columns 0..127), each on its
        // TMEM lane quarter; the accumulator is released as soon as both
        // maxima are in registers.
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32);
        const bool near = warp < 6;
        // max over one 128-key block, read from TMEM in two halves of 64
        // columns (14 warps leave 128 registers a thread); the own block is
        // cut at the query (causal)
        auto block_max = [&](uint32_t ta, bool diag) -> float {
            float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
            // four quarters of 32 columns, the next quarter's load in flight
            // while one is reduced
            uint32_t va[32], vb[32];
            tmem_ld32(ta, va);
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) {
                uint32_t* v = (qd & 1) ? vb : va;
                tmem_ld_wait_regs(v);
                if (qd + 1 < 4) tmem_ld32(ta + (qd + 1) * 32, (qd & 1) ? va : vb);
                if (diag) {
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (qd * 32 + c > r) v[c] = __float_as_uint(-INFINITY);
                }
#pragma unroll
                for (int c = 0; c < 32; c += 8) {
                    m0 = fmax3(m0, __uint_as_float(v[c + 0]), __uint_as_float(v[c + 1]));
                    m1 = fmax3(m1, __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
                    m2 = fmax3(m2, __uint_as_float(v[c + 4]), __uint_as_float(v[c + 5]));
                    m3 = fmax3(m3, __uint_as_float(v[c + 6]), __uint_as_float(v[c + 7]));
                }
            }
            return fmaxf(fmax3(m0, m1, m2), m3);
        };
        for (int k = 0; k < npairs; ++k) {
            const int hi = ntiles - 1 - 2 * k, lo = hi - 1;
            const int buf = k % NACC;
            bool ok = mbar_wait(&acc_full[buf], (uint32_t)(k / NACC) & 1u, wc, code0 + 4);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t ta = tmem_addr(tmem, lane_base, (uint32_t)buf * 256u);
            const float mx = near ? block_max(ta + 128, hi == qb) : (lo >= 0 ? block_max(ta, false) : -INFINITY);
            tc_fence_before();
            mbar_arrive(&acc_empty[buf]);   // the accumulator is free for pair k + NACC
            const int slot = k % ring;
            if (k >= ring) {
                ok = mbar_wait(&pm_empty[slot], (uint32_t)(k / ring - 1) & 1u, wc, code0 + 5);
                if (!__all_sync(0xffffffffu, ok)) break;
            }
            pm[(slot * 2 + (near ? 1 : 0)) * 128 + r] = mx;
            mbar_arrive(&pm_full[slot]);
        }
    } else {
        // ---------------- selection: rows 32 (warp - 10) .. + 31 ----------------
        int cnt = 0, npend = 0;
        float tau = -INFINITY;   // score of the heap root once the heap is full
        auto merge_pending = [&]() {
            for (int e = 0; e < npend; ++e) {
                const uint2 c = pend[e * 128 + r];
                if (__uint_as_float(c.x) >= __uint_as_float(heap[r].x)) {   // lower id than every kept
                    heap[r] = c;                                            // pair: ties go to it
                    sift_down(heap, k1, r, 0);
                }
            }
            npend = 0;
            tau = __uint_as_float(heap[r].x);
        };
        // blocks arrive in descending order: the next forced block below the own
        // one is a running pointer (-1 once all nf - 1 of them have passed)
        int next_forced = nf > 1 ? qb - p.dilation : -1, forced_left = nf - 1;
        auto consume = [&](int n, float mx) {
            if (dbg && row_ok) p.pooled[((int64_t)bg * p.T + i) * p.nblk + n] = mx;
            if (!need_heap || n == qb) return;
            if (WINDOW && n == next_forced) {   // forced: kept without ranking
                next_forced = --forced_left > 0 ? n - p.dilation : -1;
                return;
            }
            if (cnt < k1) {   // same count for every row of the tile: warp-uniform
                heap[cnt * 128 + r] = cand(mx, n);
                if (++cnt == k1) {
                    for (int x = (k1 - 2) / 4; x >= 0; --x) sift_down(heap, k1, r, x);
                    tau = __uint_as_float(heap[r].x);
                }
            } else if (mx >= tau) {
                pend[npend * 128 + r] = cand(mx, n);
                ++npend;
            }
        };
        // two pairs per handshake: both slots' maxima are read together
        for (int k = 0; k < npairs; k += 2) {
            const bool two = k + 1 < npairs;
            const int hi = ntiles - 1 - 2 * k, lo = hi - 1;
            const int slot = k % ring, slot1 = (k + 1) % ring;
            bool ok = mbar_wait(&pm_full[slot], (uint32_t)(k / ring) & 1u, wc, code0 + 6);
            if (ok && two) ok = mbar_wait(&pm_full[slot1], (uint32_t)((k + 1) / ring) & 1u, wc, code0 + 6);
            if (!__all_sync(0xffffffffu, ok)) break;
            const float mhi = pm[(slot * 2 + 1) * 128 + r], mlo = pm[slot * 2 * 128 + r];
            const float mhi1 = two ? pm[(slot1 * 2 + 1) * 128 + r] : 0.f, mlo1 = two ? pm[slot1 * 2 * 128 + r] : 0.f;
            mbar_arrive(&pm_empty[slot]);
            if (two) mbar_arrive(&pm_empty[slot1]);
            consume(hi, mhi);
            if (lo >= 0) consume(lo, mlo);
            if (two) {
                consume(hi - 2, mhi1);
                if (lo - 2 >= 0) consume(lo - 2, mlo1);
            }
            // one vote per two pairs: at most four appends, so a list holding
            // 6 still has room for the next two pairs
            if (need_heap && cnt == k1 && __any_sync(0xffffffffu, npend >= kPend - 4)) merge_pending();
        }
        if (need_heap && cnt == k1) merge_pending();
        const bool go = __all_sync(0xffffffffu, !*abort_flag);
        __syncwarp();   // each lane's heap column is read by the whole warp below
        if (go) {
            if (need_heap) {
                // every MMA has finished (the last pair's maxima have been
                // read), so the key ring is free to stage the sorted rows
                const int64_t row0 = (int64_t)bg * p.T + qb * 128;
                int32_t* stg = (int32_t*)kp_tiles;
                if (p.topk <= 32)
                    write_selection_rows<32>(heap, k1, p.topk, p.dilation, warp - 10, qb, p.T, row0, p.idx, p.nsel,
                                             stg);
                else if (p.topk <= 64)
                    write_selection_rows<64>(heap, k1, p.topk, p.dilation, warp - 10, qb, p.T, row0, p.idx, p.nsel,
                                             stg);
                else
                    write_selection<4>(heap, k1, p.topk, p.dilation, warp - 10, qb, p.T, row0, p.idx, p.nsel);
            } else if (row_ok) {
                write_unranked(p.idx + ((int64_t)bg * p.T + i) * p.topk, p.nsel + (int64_t)bg * p.T + i, take_all,
                               qb, nf, p.dilation, p.topk);
            }
            if (dbg && row_ok)
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

template <int NSTAGE, int RING, bool WINDOW>
cudaError_t launch_variant(const Problem& pr, const CUtensorMap& tm_qp, const CUtensorMap& tm_kp,
                           const Params& p, size_t smem, cudaStream_t st)
{
    auto kern = proxy_select_kernel<NSTAGE, RING, WINDOW>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((pr.nblk - pr.qb0) * pr.B * pr.Hp);
    trace_begin(kTraceProxy, st);
    kern<<<grid, kThreads, smem, st>>>(tm_qp, tm_kp, p);
    count_launches(1);
    trace_end(kTraceProxy, st);
    return cudaGetLastError();
}

size_t smem_bytes(int nstage, int topk, int ring)
{
    const size_t k1 = (size_t)(topk > 1 ? topk - 1 : 0);
    return 1024 + (size_t)kTileBytes * (1 + 2 * nstage) + k1 * 128 * 8 + (size_t)kPend * 128 * 8 +
           (size_t)ring * 2 * 128 * 4 + (size_t)(2 * nstage + 2 * kNacc + 2 * ring + 2) * 8 + 16;
}

}  // namespace

cudaError_t launch_proxy_select(const Problem& pr, const CUtensorMap& tm_qp, const CUtensorMap& tm_kp,
                                int32_t* idx, int32_t* nsel, float* pooled, uint32_t* status,
                                cudaStream_t st)
{
    Params p{pr.B, pr.T, pr.Hp, pr.dp, pr.nblk, pr.topk, pr.qb0, pr.window, pr.dilation, idx, nsel, pooled, status};
    // Shared memory is split between key stages and the maxima ring: three
    // stages and a 40-slot ring while topk leaves room for them (the deep ring
    // absorbs the selection's merge bursts: 4.5 % faster at 128K than four
    // stages and 8 slots), else two stages and 8 slots.  All of TMEM per CTA:
    // at least 120 KB of shared memory keeps one CTA per SM.
    const bool win = pr.window > 1;
    const size_t deep = smem_bytes(3, pr.topk, 40);
    if (deep <= 227 * 1024) {
        const size_t sm = deep < 120 * 1024 ? 120 * 1024 : deep;
        return win ? launch_variant<3, 40, true>(pr, tm_qp, tm_kp, p, sm, st)
                   : launch_variant<3, 40, false>(pr, tm_qp, tm_kp, p, sm, st);
    }
    const size_t small = smem_bytes(2, pr.topk, 8);
    if (small > 227 * 1024) return cudaErrorInvalidValue;
    const size_t sm = small < 120 * 1024 ? 120 * 1024 : small;
    return win ? launch_variant<2, 8, true>(pr, tm_qp, tm_kp, p, sm, st)
               : launch_variant<2, 8, false>(pr, tm_qp, tm_kp, p, sm, st);
}

}  // namespace msa
