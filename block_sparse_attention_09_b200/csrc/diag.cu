// Diagnostics used by the GPU tests (no counterpart in the method):
//  * diag_umma_kernel: one 128 x N x K tcgen05 MMA with the operands staged
//    in each of the ways the real kernels stage them (K-major or MN-major
//    128-byte-swizzled shared memory, or A in tensor memory), so the layout
//    conventions can be checked against a plain matrix product.
//  * diag_wait_kernel: an mbarrier wait that nothing completes; the bounded
//    wait must give up, record MSA_ERR_TIMEOUT in the status word and return.
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

// mode: 0 A,B K-major | 1 A K-major, B MN-major | 2 A,B MN-major |
//       3 A TMEM, B MN-major | 4 A TMEM, B K-major.
__global__ void __launch_bounds__(128, 1) diag_umma_kernel(int mode, int N, int K,
                                                           const __nv_bfloat16* __restrict__ A,
                                                           const __nv_bfloat16* __restrict__ B,
                                                           float* __restrict__ D, uint32_t* status)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* a_tile = smem;             // up to 128 x 128 bf16 (32 KB)
    uint8_t* b_tile = smem + 32768;     // up to 128 x 128 bf16
    uint64_t* bar = (uint64_t*)(smem + 65536 + 32768);   // 32 KB gap: reads past a tile stay inside
    uint32_t* tmem_hold = (uint32_t*)(bar + 1);
    volatile uint32_t* abort_flag = tmem_hold + 1;
    const int t = threadIdx.x, warp = t >> 5;
    const bool a_tmem = mode >= 3;
    const bool a_mn = mode == 2;
    const bool b_mn = mode == 1 || mode == 2 || mode == 3;

    if (t == 0) {
        mbar_init(bar, 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(tmem_hold, 256); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_hold;   // D at columns [0, N), A at [128, 128 + K/2)

    // ---- stage A row t ----
    if (a_tmem) {
        for (int c0 = 0; c0 < K / 2; c0 += 16) {
            uint32_t pk[16];
            for (int e = 0; e < 16; ++e) {
                const int kk = 2 * (c0 + e);
                pk[e] = pack_bf16x2(__bfloat162float(A[t * K + kk]), __bfloat162float(A[t * K + kk + 1]));
            }
            tmem_st16(tmem_addr(tmem, (uint32_t)warp * 32u, 128u + c0), pk);
        }
        tmem_st_wait();
    } else if (!a_mn) {
        const uint32_t base = smem_u32(a_tile);
        for (int ch = 0; ch < K / 8; ++ch) {
            uint4 u = *reinterpret_cast<const uint4*>(A + t * K + ch * 8);
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(base + sw128_offset(t, ch & 7, ch >> 3, 128)),
                         "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w) : "memory");
        }
    } else {
        // physical [K rows][128 M columns]: element (m = t, k) at row k, column t
        __nv_bfloat16* tile = (__nv_bfloat16*)a_tile;
        for (int k = 0; k < K; ++k) {
            const uint32_t off = sw128_offset(k, (t & 63) >> 3, t >> 6, K);
            tile[(off >> 1) + (t & 7)] = A[t * K + k];
        }
    }
    // ---- stage B row t (t < N) ----
    if (t < N) {
        if (!b_mn) {
            const uint32_t base = smem_u32(b_tile);
            for (int ch = 0; ch < K / 8; ++ch) {
                uint4 u = *reinterpret_cast<const uint4*>(B + t * K + ch * 8);
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(base + sw128_offset(t, ch & 7, ch >> 3, N)),
                             "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w) : "memory");
            }
        } else {
            __nv_bfloat16* tile = (__nv_bfloat16*)b_tile;
            for (int k = 0; k < K; ++k) {
                const uint32_t off = sw128_offset(k, (t & 63) >> 3, t >> 6, K);
                tile[(off >> 1) + (t & 7)] = B[t * K + k];
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (t == 0) {
        const uint32_t idesc = idesc_bf16(128, (uint32_t)N, a_mn, b_mn);
        const uint32_t aa = smem_u32(a_tile), ba = smem_u32(b_tile);
        for (int kk = 0; kk < K / 16; ++kk) {
            uint64_t bd;
            if (!b_mn) bd = desc_kmajor(ba, (uint32_t)N, kk * 16);
            else bd = desc_mnmajor(ba, (uint32_t)K, kk * 16);
            if (a_tmem) {
                umma_ts(tmem, tmem + 128u + kk * 8, bd, idesc, kk > 0 ? 1u : 0u);
            } else {
                uint64_t ad;
                if (!a_mn) ad = desc_kmajor(aa, 128, kk * 16);
                else ad = desc_mnmajor(aa, (uint32_t)K, kk * 16);
                umma_ss(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
        }
        umma_commit(bar);
    }
    const WaitCtx wc{status, abort_flag, 1000000000ull};
    const bool ok = mbar_wait(bar, 0, wc, kStTimeoutBase + kKidDiag * 16);
    if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        for (int c0 = 0; c0 < N; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem_addr(tmem, (uint32_t)warp * 32u, (uint32_t)c0), v);
            tmem_ld_wait();
            for (int e = 0; e < 32; ++e) D[t * N + c0 + e] = __uint_as_float(v[e]);
        }
    } else if (t == 0) {
        mbar_drain(bar, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

__global__ void diag_wait_kernel(uint64_t limit_ns, uint32_t* status)
{
    __shared__ uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0u;
        fence_mbar_init();
    }
    __syncthreads();
    const WaitCtx wc{status, &abort_flag, limit_ns};
    // nothing ever arrives on this barrier: the wait must give up by itself
    mbar_wait(&bar, 0, wc, kStTimeoutBase + kKidDiag * 16 + 1);
}

}  // namespace

cudaError_t launch_diag_umma(int mode, int N, int K, const void* A, const void* B, float* D,
                             uint32_t* status, cudaStream_t st)
{
    const size_t smem = 1024 + 65536 + 32768 + 64;
    cudaError_t e = cudaFuncSetAttribute(diag_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    diag_umma_kernel<<<1, 128, smem, st>>>(mode, N, K, (const __nv_bfloat16*)A, (const __nv_bfloat16*)B,
                                           D, status);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_diag_wait(uint64_t limit_ns, uint32_t* status, cudaStream_t st)
{
    diag_wait_kernel<<<1, 32, 0, st>>>(limit_ns, status);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace msa
