// Block -> query inverse index of the cached block selection.
//
// The Main Branch kernels are KV-stationary: one CTA owns one KV block of
// one group and streams the queries that selected it.  This file turns the
// per-query selection idx[b,g,i,:] into, for every (b, g, block n), the
// ascending list of query positions i whose selection holds n (CSR:
// ptr[bg][n] .. ptr[bg][n+1] into tok[bg][...]).
//
// Deterministic construction (no atomics on the output order):
//   count: per (bg, query tile qb) a 128-bit membership mask per block n
//          in shared memory -> cnt[bg][qb][n] = popcount
//   scan:  exclusive prefix of cnt over qb for each n (in place) and the
//          total per n
//   ptr:   exclusive prefix of the totals over n
//   fill:  rebuild the masks; query t of tile qb writes itself at
//          ptr[n] + cnt[qb][n] + popcount(mask bits below t)
// The same construction also yields the PAIR index the forward reads: for
// every (b, g, pair p = blocks 2p and 2p+1), the ascending list of queries
// that selected either block, each entry (i << 2) | bit0 (selected 2p) |
// bit1 (selected 2p+1).  A query that selected both blocks appears once.
// Selection entries outside [0, i/128], not strictly ascending, or rows
// with nsel outside [1, topk] are skipped and flagged in the status word.
// Only query tiles qb0 .. nblk-1 take part (rows before the first computed
// query are not read): their cnt rows alone are written and scanned.
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

// Membership word w (0..3) of the union of blocks 2p and 2p+1 in a tile
// whose masks cover blocks 0 .. qb (blocks past qb are selected by no query
// of the tile).
__device__ __forceinline__ uint32_t pair_word(const uint32_t* mask, int p, int qb, int w)
{
    return mask[(2 * p) * 4 + w] | (2 * p + 1 <= qb ? mask[(2 * p + 1) * 4 + w] : 0u);
}

__global__ void __launch_bounds__(128) index_count_kernel(const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ nsel, int T, int topk,
                                                          int nblk, int npair, int qb0, int32_t* __restrict__ cnt,
                                                          int32_t* __restrict__ cnt2, uint32_t* status)
{
    extern __shared__ uint32_t mask[];
    const int qb = qb0 + (int)blockIdx.x, bg = blockIdx.y;
    if (!build_masks(mask, idx, nsel, T, topk, qb, bg)) atomicOr(status + 1, 1u);
    int32_t* out = cnt + ((int64_t)bg * nblk + qb) * nblk;
    for (int n = threadIdx.x; n <= qb; n += blockDim.x)
        out[n] = __popc(mask[n * 4]) + __popc(mask[n * 4 + 1]) + __popc(mask[n * 4 + 2]) +
                 __popc(mask[n * 4 + 3]);
    int32_t* out2 = cnt2 + ((int64_t)bg * nblk + qb) * npair;
    for (int p = threadIdx.x; 2 * p <= qb; p += blockDim.x)
        out2[p] = __popc(pair_word(mask, p, qb, 0)) + __popc(pair_word(mask, p, qb, 1)) +
                  __popc(pair_word(mask, p, qb, 2)) + __popc(pair_word(mask, p, qb, 3));
}

// cnt[bg][qb][n] (ncols columns) for qb >= max(cstep * n, qb0)  ->
// exclusive prefix over qb; tot[bg][n] = sum.  cstep = 1: block columns;
// cstep = 2: pair columns (pair n is first selectable from tile 2n).
// Block (32 x 32): x = column within a group of 32, y = segment of qb;
// gridDim.z = 2 runs the block matrix (z = 0) and the pair matrix (z = 1).
__global__ void __launch_bounds__(1024) index_scan_kernel(int32_t* __restrict__ cnt, int32_t* __restrict__ tot,
                                                          int32_t* __restrict__ cnt2, int32_t* __restrict__ tot2,
                                                          int nblk, int npair, int qb0)
{
    __shared__ int seg[32][33];
    const bool pairs = blockIdx.z == 1;
    const int ncols = pairs ? npair : nblk, cstep = pairs ? 2 : 1;
    int32_t* const m = pairs ? cnt2 : cnt;
    int32_t* const t = pairs ? tot2 : tot;
    const int n0 = blockIdx.x * 32;
    if (n0 >= ncols) return;                         // block-uniform
    const int n = n0 + threadIdx.x, bg = blockIdx.y;
    const int r0 = min(cstep * n0, nblk);            // rows qb in [r0, nblk) cover every column here
    const int per = (nblk - r0 + 31) / 32;
    const int q0 = r0 + threadIdx.y * per;
    const int q1 = min(q0 + per, nblk);
    int32_t* col = m + (int64_t)bg * nblk * ncols + n;
    int s = 0;
    if (n < ncols)
        for (int q = max(q0, max(cstep * n, qb0)); q < q1; ++q) s += col[(int64_t)q * ncols];
    seg[threadIdx.y][threadIdx.x] = s;
    __syncthreads();
    int base = 0;
    for (int y = 0; y < (int)threadIdx.y; ++y) base += seg[y][threadIdx.x];
    if (n < ncols) {
        int run = base;
        for (int q = max(q0, max(cstep * n, qb0)); q < q1; ++q) {
            const int c = col[(int64_t)q * ncols];
            col[(int64_t)q * ncols] = run;
            run += c;
        }
        if (threadIdx.y == 31) t[(int64_t)bg * ncols + n] = base + s;
    }
}

// ptr[bg][0..nblk] = exclusive prefix of tot[bg][0..nblk) (blockIdx.y = 0),
// ptr2[bg][0..npair] of tot2 (blockIdx.y = 1).
__global__ void __launch_bounds__(1024) index_ptr_kernel(const int32_t* __restrict__ tot1,
                                                         int32_t* __restrict__ ptr1, const int32_t* __restrict__ tot2,
                                                         int32_t* __restrict__ ptr2, int nblk1, int npair)
{
    __shared__ int part[1024];
    const bool pairs = blockIdx.y == 1;
    const int32_t* tot = pairs ? tot2 : tot1;
    int32_t* ptr = pairs ? ptr2 : ptr1;
    const int nblk = pairs ? npair : nblk1;
    const int bg = blockIdx.x, t = threadIdx.x;
    const int per = (nblk + 1023) / 1024;
    const int a0 = t * per, a1 = min(a0 + per, nblk);
    const int32_t* in = tot + (int64_t)bg * nblk;
    int32_t* out = ptr + (int64_t)bg * (nblk + 1);
    int s = 0;
    for (int a = a0; a < a1; ++a) s += in[a];
    part[t] = s;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {    // inclusive Hillis-Steele scan
        const int v = t >= off ? part[t - off] : 0;
        __syncthreads();
        part[t] += v;
        __syncthreads();
    }
    int run = part[t] - s;
    for (int a = a0; a < a1; ++a) { out[a] = run; run += in[a]; }
    if (t == 1023) out[nblk] = part[1023];
}

// The tile's queries that selected block n form one run of the block's token
// list (ptr[n] + off[qb][n] onward), in ascending order: a warp writes it
// from the tile's membership mask, lane l taking bit l of each 32-bit word, so
// the stores of one word land on consecutive positions.
__global__ void __launch_bounds__(512) index_fill_kernel(const int32_t* __restrict__ idx,
                                                         const int32_t* __restrict__ nsel, int T, int topk,
                                                         int nblk, int npair, int qb0, const int32_t* __restrict__ off,
                                                         const int32_t* __restrict__ ptr, int32_t* __restrict__ tok,
                                                         const int32_t* __restrict__ off2,
                                                         const int32_t* __restrict__ ptr2,
                                                         int32_t* __restrict__ tok2)
{
    extern __shared__ uint32_t mask[];
    const int qb = qb0 + (int)blockIdx.x, bg = blockIdx.y;
    build_masks(mask, idx, nsel, T, topk, qb, bg);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = (int)(blockDim.x >> 5);
    const uint32_t below = (1u << lane) - 1u;
    // A warp takes 32 consecutive blocks at a time: their list offsets are
    // loaded together (lane j: block n0 + j, one coalesced load each), so the
    // per-block loop below runs on shared memory and shuffles only.
    {
        const int32_t* offrow = off + ((int64_t)bg * nblk + qb) * nblk;
        const int32_t* p = ptr + (int64_t)bg * (nblk + 1);
        int32_t* out = tok + (int64_t)bg * T * topk;
        for (int n0 = warp * 32; n0 <= qb; n0 += nwarps * 32) {
            const int nl = n0 + lane;
            const int base = nl <= qb ? p[nl] + offrow[nl] : 0;
            const int nn = min(32, qb + 1 - n0);
            for (int j = 0; j < nn; ++j) {
                const int n = n0 + j;
                const uint32_t m0 = mask[n * 4], m1 = mask[n * 4 + 1], m2 = mask[n * 4 + 2], m3 = mask[n * 4 + 3];
                int pos = __shfl_sync(0xffffffffu, base, j);
                if ((m0 | m1 | m2 | m3) == 0u) continue;
                const uint32_t mw[4] = {m0, m1, m2, m3};
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    if ((mw[w] >> lane) & 1u) out[pos + __popc(mw[w] & below)] = qb * 128 + w * 32 + lane;
                    pos += __popc(mw[w]);
                }
            }
        }
    }
    // pair lists: the union of blocks 2p and 2p+1, with per-entry flags
    const int32_t* offrow = off2 + ((int64_t)bg * nblk + qb) * npair;
    const int32_t* p = ptr2 + (int64_t)bg * (npair + 1);
    int32_t* out = tok2 + (int64_t)bg * T * topk;
    for (int p0 = warp * 32; 2 * p0 <= qb; p0 += nwarps * 32) {
        const int pl = p0 + lane;
        const int base = 2 * pl <= qb ? p[pl] + offrow[pl] : 0;
        const int nn = min(32, qb / 2 + 1 - p0);
        for (int j = 0; j < nn; ++j) {
            const int pp = p0 + j;
            uint32_t a[4], c[4], u = 0u;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                a[w] = mask[(2 * pp) * 4 + w];
                c[w] = 2 * pp + 1 <= qb ? mask[(2 * pp + 1) * 4 + w] : 0u;
                u |= a[w] | c[w];
            }
            int pos = __shfl_sync(0xffffffffu, base, j);
            if (u == 0u) continue;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t mw = a[w] | c[w];
                if ((mw >> lane) & 1u)
                    out[pos + __popc(mw & below)] = ((qb * 128 + w * 32 + lane) << 2) | (int)((a[w] >> lane) & 1u) |
                                                    (int)(((c[w] >> lane) & 1u) << 1);
                pos += __popc(mw);
            }
        }
    }
}

}  // namespace

cudaError_t launch_block_index(const Problem& pr, const int32_t* idx, const int32_t* nsel, void* ws,
                               const WsLayout& L, cudaStream_t st)
{
    uint8_t* w = (uint8_t*)ws;
    int32_t* cnt = (int32_t*)(w + L.cnt);
    int32_t* tot = (int32_t*)(w + L.tot);
    int32_t* ptr = (int32_t*)(w + L.ptr);
    int32_t* tok = (int32_t*)(w + L.tok);
    int32_t* cnt2 = (int32_t*)(w + L.cnt2);
    int32_t* tot2 = (int32_t*)(w + L.tot2);
    int32_t* ptr2 = (int32_t*)(w + L.ptr2);
    int32_t* tok2 = (int32_t*)(w + L.tok2);
    uint32_t* status = (uint32_t*)(w + L.status);
    const int BH = pr.B * pr.Hp;
    const int npair = pair_count(pr.nblk);
    const size_t mask_bytes = (size_t)pr.nblk * 16;
    if (mask_bytes > 48 * 1024) {
        cudaError_t e;
        e = cudaFuncSetAttribute(index_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)mask_bytes);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(index_fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)mask_bytes);
        if (e != cudaSuccess) return e;
    }
    dim3 g1(pr.nblk - pr.qb0, BH);   // the computed query tiles
    index_count_kernel<<<g1, 128, mask_bytes, st>>>(idx, nsel, pr.T, pr.topk, pr.nblk, npair, pr.qb0, cnt, cnt2,
                                                    status);
    count_launches(1);
    dim3 g2((pr.nblk + 31) / 32, BH, 2), b2(32, 32);
    index_scan_kernel<<<g2, b2, 0, st>>>(cnt, tot, cnt2, tot2, pr.nblk, npair, pr.qb0);
    count_launches(1);
    index_ptr_kernel<<<dim3(BH, 2), 1024, 0, st>>>(tot, ptr, tot2, ptr2, pr.nblk, npair);
    count_launches(1);
    index_fill_kernel<<<g1, 512, mask_bytes, st>>>(idx, nsel, pr.T, pr.topk, pr.nblk, npair, pr.qb0, cnt, ptr, tok,
                                                   cnt2, ptr2, tok2);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace msa
