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
// Selection entries outside [0, i/128], not strictly ascending, or rows
// with nsel outside [1, topk] are skipped and flagged in the status word.
// Only query tiles qb0 .. nblk-1 take part (rows before the first computed
// query are not read): their cnt rows alone are written and scanned.
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

// Shared masks of one query tile, returns false on a malformed row.
__device__ bool build_masks(uint32_t* mask, const int32_t* idx, const int32_t* nsel, int T, int topk,
                            int qb, int bg)
{
    const int nb = qb + 1;
    for (int x = threadIdx.x; x < nb * 4; x += blockDim.x) mask[x] = 0u;
    __syncthreads();
    bool bad = false;
    const int t = threadIdx.x, i = qb * 128 + t;
    if (t < 128 && i < T) {
        const int64_t row = (int64_t)bg * T + i;
        int ns = nsel[row];
        if (ns < 1 || ns > topk) { bad = true; ns = ns < 0 ? 0 : (ns > topk ? topk : ns); }
        const int32_t* sel = idx + row * topk;
        int prev = -1;
        for (int s = 0; s < ns; ++s) {
            const int n = sel[s];
            if (n < 0 || n > qb || n <= prev) { bad = true; continue; }
            prev = n;
            atomicOr(&mask[n * 4 + (t >> 5)], 1u << (t & 31));
        }
    }
    __syncthreads();
    return !bad;
}

__global__ void __launch_bounds__(128) index_count_kernel(const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ nsel, int T, int topk,
                                                          int nblk, int qb0, int32_t* __restrict__ cnt,
                                                          uint32_t* status)
{
    extern __shared__ uint32_t mask[];
    const int qb = qb0 + (int)blockIdx.x, bg = blockIdx.y;
    if (!build_masks(mask, idx, nsel, T, topk, qb, bg)) atomicOr(status + 1, 1u);
    int32_t* out = cnt + ((int64_t)bg * nblk + qb) * nblk;
    for (int n = threadIdx.x; n <= qb; n += blockDim.x)
        out[n] = __popc(mask[n * 4]) + __popc(mask[n * 4 + 1]) + __popc(mask[n * 4 + 2]) +
                 __popc(mask[n * 4 + 3]);
}

// cnt[bg][qb][n] for qb >= max(n, qb0)  ->  exclusive prefix over qb;
// tot[bg][n] = sum.  Block (32 x 32): x = block id within a group of 32,
// y = segment of qb.
__global__ void __launch_bounds__(1024) index_scan_kernel(int32_t* __restrict__ cnt,
                                                          int32_t* __restrict__ tot, int nblk, int qb0)
{
    __shared__ int seg[32][33];
    const int n0 = blockIdx.x * 32;
    const int n = n0 + threadIdx.x, bg = blockIdx.y;
    const int len = nblk - n0;                       // rows qb in [n0, nblk) cover every n here
    const int per = (len + 31) / 32;
    const int q0 = n0 + threadIdx.y * per;
    const int q1 = min(q0 + per, nblk);
    int32_t* col = cnt + (int64_t)bg * nblk * nblk + n;
    int s = 0;
    if (n < nblk)
        for (int q = max(q0, max(n, qb0)); q < q1; ++q) s += col[(int64_t)q * nblk];
    seg[threadIdx.y][threadIdx.x] = s;
    __syncthreads();
    int base = 0;
    for (int y = 0; y < (int)threadIdx.y; ++y) base += seg[y][threadIdx.x];
    if (n < nblk) {
        int run = base;
        for (int q = max(q0, max(n, qb0)); q < q1; ++q) {
            const int c = col[(int64_t)q * nblk];
            col[(int64_t)q * nblk] = run;
            run += c;
        }
        if (threadIdx.y == 31) tot[(int64_t)bg * nblk + n] = base + s;
    }
}

// ptr[bg][0..nblk] = exclusive prefix of tot[bg][0..nblk).
__global__ void __launch_bounds__(1024) index_ptr_kernel(const int32_t* __restrict__ tot,
                                                         int32_t* __restrict__ ptr, int nblk)
{
    __shared__ int part[1024];
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
__global__ void __launch_bounds__(128) index_fill_kernel(const int32_t* __restrict__ idx,
                                                         const int32_t* __restrict__ nsel, int T, int topk,
                                                         int nblk, int qb0, const int32_t* __restrict__ off,
                                                         const int32_t* __restrict__ ptr,
                                                         int32_t* __restrict__ tok)
{
    extern __shared__ uint32_t mask[];
    const int qb = qb0 + (int)blockIdx.x, bg = blockIdx.y;
    build_masks(mask, idx, nsel, T, topk, qb, bg);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t* offrow = off + ((int64_t)bg * nblk + qb) * nblk;
    const int32_t* p = ptr + (int64_t)bg * (nblk + 1);
    int32_t* out = tok + (int64_t)bg * T * topk;
    const uint32_t below = (1u << lane) - 1u;
    for (int n = warp; n <= qb; n += 4) {
        const uint32_t m0 = mask[n * 4], m1 = mask[n * 4 + 1], m2 = mask[n * 4 + 2], m3 = mask[n * 4 + 3];
        if ((m0 | m1 | m2 | m3) == 0u) continue;
        int pos = p[n] + offrow[n];
        const uint32_t mw[4] = {m0, m1, m2, m3};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            if ((mw[w] >> lane) & 1u) out[pos + __popc(mw[w] & below)] = qb * 128 + w * 32 + lane;
            pos += __popc(mw[w]);
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
    uint32_t* status = (uint32_t*)(w + L.status);
    const int BH = pr.B * pr.Hp;
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
    index_count_kernel<<<g1, 128, mask_bytes, st>>>(idx, nsel, pr.T, pr.topk, pr.nblk, pr.qb0, cnt, status);
    count_launches(1);
    dim3 g2((pr.nblk + 31) / 32, BH), b2(32, 32);
    index_scan_kernel<<<g2, b2, 0, st>>>(cnt, tot, pr.nblk, pr.qb0);
    count_launches(1);
    index_ptr_kernel<<<BH, 1024, 0, st>>>(tot, ptr, pr.nblk);
    count_launches(1);
    index_fill_kernel<<<g1, 128, mask_bytes, st>>>(idx, nsel, pr.T, pr.topk, pr.nblk, pr.qb0, cnt, ptr, tok);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace msa
