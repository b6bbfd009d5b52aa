// Device-side building blocks for the sm_100a kernels: mbarriers with bounded
// waits, TMA tile loads, cp.async gathers, tcgen05 (TMEM alloc / MMA / commit /
// ld / st) and the UMMA shared-memory and instruction descriptors.
//
// Every wait in this library is bounded: after MSA_WAIT_LIMIT_NS without
// progress it records an error code in the caller's status word, raises the
// CTA's abort flag so that every other wait of the CTA gives up at once, and
// returns false.  Kernels then unwind, drain their own copies / MMAs with a
// short bounded wait, free TMEM and exit.  Nothing traps.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define MSA_DEV __device__ __forceinline__

#ifndef MSA_WAIT_LIMIT_NS
#define MSA_WAIT_LIMIT_NS 4000000000ull   // 4 s without progress = failure
#endif
#define MSA_DRAIN_LIMIT_NS 100000000ull   // 100 ms for teardown drains

namespace msa {

// ---------------------------------------------------------------- basics
MSA_DEV uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

MSA_DEV uint64_t global_timer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

MSA_DEV uint32_t lane_id() { return threadIdx.x & 31u; }

MSA_DEV void named_bar_sync(uint32_t id, uint32_t nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ANDs a predicate over the participating threads:
// every thread learns whether all of them may go on, so a group never splits
// into threads that leave and threads that wait at a later barrier.
MSA_DEV bool bar_and_sync(uint32_t id, uint32_t nthreads, bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0u;
}

MSA_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------- wait context
struct WaitCtx {
    uint32_t* status;              // global status word of this call
    volatile uint32_t* abort_flag; // shared: set once any wait of the CTA failed
    uint64_t limit_ns;             // give up after this long without progress
};

// ---------------------------------------------------------------- mbarrier
MSA_DEV void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

MSA_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

MSA_DEV void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

MSA_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

MSA_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.
MSA_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w, uint32_t code)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer();
    for (;;) {
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*w.abort_flag) return false;
        if (global_timer() - t0 > w.limit_ns) {
            *w.abort_flag = 1u;
            atomicCAS(w.status, 0u, code);
            return false;
        }
    }
}

// Short bounded wait used only while tearing down; ignores the abort flag.
MSA_DEV bool mbar_drain(uint64_t* bar, uint32_t parity)
{
    const uint64_t t0 = global_timer();
    while (!mbar_try_wait(bar, parity))
        if (global_timer() - t0 > MSA_DRAIN_LIMIT_NS) return false;
    return true;
}

// ---------------------------------------------------------------- TMA
MSA_DEV void tma_prefetch_desc(const CUtensorMap* map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

MSA_DEV void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                         int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// ---------------------------------------------------------------- cp.async (16 B)
// src_bytes = 0 zero-fills the destination without reading the source.
MSA_DEV void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
MSA_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
MSA_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ---------------------------------------------------------------- UMMA layout
// Operand tiles use the 128-byte swizzle canonical layout: the tile is split
// into slabs of 64 bf16 columns (128 B per row); inside a slab row r occupies
// bytes [r*128, r*128+128) and its 16-byte chunk c is stored at chunk c^(r&7).
// The same physical layout serves as a K-major operand (rows = M or N,
// columns = K) or as an MN-major operand (rows = K, columns = M or N).
MSA_DEV uint32_t sw128_offset(uint32_t row, uint32_t chunk16, uint32_t slab, uint32_t rows_per_slab)
{
    return slab * rows_per_slab * 128u + row * 128u + (((chunk16 ^ (row & 7u)) & 7u) << 4);
}

// Shared-memory matrix descriptor (sm_100 format, version 1, SWIZZLE_128B).
MSA_DEV uint64_t umma_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version for sm_100
    d |= (uint64_t)2 << 61;   // layout: 128-byte swizzle
    return d;
}

// K-major operand: rows of the tile are M (or N), K runs along the row.
// k_elem is the first K element of this MMA step (multiple of 16).
MSA_DEV uint64_t desc_kmajor(uint32_t tile_saddr, uint32_t rows, uint32_t k_elem)
{
    const uint32_t slab = k_elem >> 6, within = (k_elem & 63u) * 2u;
    return umma_desc(tile_saddr + slab * rows * 128u + within, 16u, 1024u);
}

// MN-major operand: rows of the tile are K, M (or N) runs along the row.
// Atoms of 64 MN-elements sit one slab apart (LBO); groups of 8 K-rows sit
// 1024 B apart (SBO).  k_elem is the first K row of this MMA step.
MSA_DEV uint64_t desc_mnmajor(uint32_t tile_saddr, uint32_t krows, uint32_t k_elem)
{
    return umma_desc(tile_saddr + k_elem * 128u, krows * 128u, 1024u);
}

// Instruction descriptor, kind::f16 with bf16 inputs and fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t M, uint32_t N, bool a_mn, bool b_mn)
{
    return (1u << 4)                    // D: f32
           | (1u << 7)                  // A: bf16
           | (1u << 10)                 // B: bf16
           | ((a_mn ? 1u : 0u) << 15)   // A major
           | ((b_mn ? 1u : 0u) << 16)   // B major
           | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// ---------------------------------------------------------------- tcgen05
MSA_DEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols)   // whole warp
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
MSA_DEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
MSA_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols)   // whole warp
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
MSA_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MSA_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T   (one thread issues)
MSA_DEV void umma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T   (one thread issues)
MSA_DEV void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}

// Arrive on an mbarrier once every MMA issued so far by this thread is done.
MSA_DEV void umma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

MSA_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
MSA_DEV void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bit, 32 consecutive columns per thread (thread t <- lane base+t).
MSA_DEV void tmem_ld32(uint32_t taddr, uint32_t* r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// tcgen05.wait::ld that also names the 32 registers a tcgen05.ld filled: the
// compiler then cannot move their uses above the wait (used where another
// load is issued between a load and the use of its registers).
MSA_DEV void tmem_ld_wait_regs(uint32_t* r)
{
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]),
                   "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
                   "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns per thread.
MSA_DEV void tmem_st16(uint32_t taddr, const uint32_t* r)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

// TMEM address of (lane, column) relative to an allocation base.
MSA_DEV uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col)
{
    return base + (lane << 16) + col;
}

// ---------------------------------------------------------------- work items
// The Main Branch kernels walk (group, query range, KV block) items: all KV
// blocks n that queries of range R (RB query blocks) may read, group by
// group and range by range, so the query-side rows they gather from and
// reduce into stay in L2 while a range is processed.  The token segment of
// an item comes from the inverse index: ptr[bg][n] starts block n's list and
// off[bg][qb][n] (valid for qb >= n) counts its tokens in query blocks
// before qb.
struct RangeItem {
    int bg, n, beg, count;   // beg: offset into the group's token list
};

__host__ __device__ inline int range_items_per_group(int nblk, int RB, int qb0)
{
    int total = 0;
    for (int R = 0; qb0 + R * RB < nblk; ++R) total += min(nblk, qb0 + (R + 1) * RB);
    return total;
}

// Ranges cover the query blocks qb0 .. nblk-1 (the queries computed); range R
// holds the items of KV blocks 0 .. qe-1.
MSA_DEV RangeItem range_item(int x, int nblk, int RB, int qb0, int per_group, const int32_t* ptr,
                             const int32_t* off)
{
    RangeItem it;
    it.bg = x / per_group;
    int rem = x % per_group, R = 0;
    for (;;) {
        const int nv = min(nblk, qb0 + (R + 1) * RB);
        if (rem < nv) break;
        rem -= nv;
        ++R;
    }
    const int n = rem, qs = qb0 + R * RB, qe = min(nblk, qb0 + (R + 1) * RB);
    const int32_t* pp = ptr + (int64_t)it.bg * (nblk + 1);
    const int32_t* o = off + (int64_t)it.bg * nblk * nblk;
    const int base = pp[n];
    const int start = qs > n ? o[(int64_t)qs * nblk + n] : 0;
    const int end = qe >= nblk ? pp[n + 1] - base : o[(int64_t)qe * nblk + n];
    it.n = n;
    it.beg = base + start;
    it.count = end - start;
    return it;
}

// The forward walks the same ranges over PAIRS of KV blocks (2p, 2p+1): range
// R holds the pairs p with 2p < qe.  The token segment comes from the pair
// index (ptr2 [bg][npair+1], off2 [bg][qb][npair], valid for qb >= 2p); it.n
// is the pair p.
__host__ __device__ inline int pair_items_per_group(int nblk, int RB, int qb0)
{
    int total = 0;
    for (int R = 0; qb0 + R * RB < nblk; ++R) total += (min(nblk, qb0 + (R + 1) * RB) + 1) / 2;
    return total;
}

MSA_DEV RangeItem pair_item(int x, int nblk, int npair, int RB, int qb0, int per_group, const int32_t* ptr2,
                            const int32_t* off2, int* qe_out)
{
    RangeItem it;
    it.bg = x / per_group;
    int rem = x % per_group, R = 0;
    for (;;) {
        const int np = (min(nblk, qb0 + (R + 1) * RB) + 1) / 2;
        if (rem < np) break;
        rem -= np;
        ++R;
    }
    const int pn = rem, qs = qb0 + R * RB, qe = min(nblk, qb0 + (R + 1) * RB);
    const int32_t* pp = ptr2 + (int64_t)it.bg * (npair + 1);
    const int32_t* o = off2 + (int64_t)it.bg * nblk * npair;
    const int base = pp[pn];
    const int start = qs > 2 * pn ? o[(int64_t)qs * npair + pn] : 0;
    const int end = qe >= nblk ? pp[pn + 1] - base : o[(int64_t)qe * npair + pn];
    it.n = pn;
    it.beg = base + start;
    it.count = end - start;
    *qe_out = qe;
    return it;
}

// Block-membership masks of one query tile in shared memory: bit t of
// mask[n*4 + t/32] says query qb*128 + t selected block n (n <= qb).  The
// whole CTA calls it; returns false on a malformed row (entries outside
// [0, i/128], not ascending, nsel outside [1, topk]), whose bad entries are
// skipped.
__device__ __forceinline__ bool build_masks(uint32_t* mask, const int32_t* idx, const int32_t* nsel, int T, int topk,
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

// Active query row r (0 .. B*(T-q0)*Hq - 1: the rows q0 .. T-1 of every batch
// and head, head fastest) -> (b, i, h).  Small: r < 2^31, so 32-bit division
// suffices (the 64-bit one costs several times as many instructions).
template <bool Small>
MSA_DEV void active_coords(int64_t r, int T, int Hq, int q0, int& b, int& i, int& h)
{
    const int Tq = T - q0;
    if (Small) {
        const uint32_t ru = (uint32_t)r, hq = (uint32_t)Hq, tq = (uint32_t)Tq;
        const uint32_t bi = ru / hq;
        h = (int)(ru - bi * hq);
        const uint32_t bb = bi / tq;
        i = q0 + (int)(bi - bb * tq);
        b = (int)bb;
    } else {
        h = (int)(r % Hq);
        const int64_t bi = r / Hq;
        i = q0 + (int)(bi % Tq);
        b = (int)(bi / Tq);
    }
}

// Active query row r (0 .. B*(T-q0)*Hq - 1: the rows q0 .. T-1 of every batch
// and head) -> its flat index (b*T + i)*Hq + h in a [B][T][Hq] tensor.
MSA_DEV int64_t active_row(int64_t r, int T, int Hq, int q0)
{
    const int h = (int)(r % Hq);
    const int64_t bi = r / Hq;
    const int Tq = T - q0;
    const int i = q0 + (int)(bi % Tq), b = (int)(bi / Tq);
    return ((int64_t)b * T + i) * Hq + h;
}

// ---------------------------------------------------------------- math
MSA_DEV float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

MSA_DEV float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

MSA_DEV uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

MSA_DEV void red_add_v4(float* gptr, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(gptr), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}

}  // namespace msa
