// Host-side declarations shared by the C-ABI layer and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace msa {

constexpr int kBlock = 128;      // KV block length of the method
constexpr int kMaxTopk = 128;    // selection heap lives in shared memory
constexpr int kMaxT = 1 << 20;   // per-tile block masks (nblk * 16 B) stay in shared memory

// Device status word codes (first word of every workspace).  The high byte
// says which kernel, the low bits which wait or check.
enum : uint32_t {
    kStOk = 0,
    kStTimeoutBase = 0x100,      // + kernel id * 16 + wait id
    kStIndexError = 0x8000,      // an idx entry outside [0, i/128]
};
enum KernelId : uint32_t { kKidProxy = 1, kKidFwd = 2, kKidBwd = 3, kKidDiag = 4 };

struct Problem {
    int B, T, Hq, Hkv, Hp, d, dp, topk, nblk, G;
    int window, dilation;   // forced block pattern of the selection (>= 1)
    int q0, qb0;            // first query row computed, and its block (q0 = 128 qb0)
    float scale;
    int64_t rows_q() const { return (int64_t)B * T * Hq; }
    // query rows computed: rows q0 .. T-1 of every batch and head
    int64_t rows_q_active() const { return (int64_t)B * (T - q0) * Hq; }
};

// Byte offsets of the workspace regions.
struct WsLayout {
    size_t status = 0;   // 256 B: [0] timeout code, [1] index error, [2] forward fallback rows
    size_t cnt = 0, tot = 0, ptr = 0, tok = 0;       // block -> query inverse index
    size_t cnt2 = 0, tot2 = 0, ptr2 = 0, tok2 = 0;   // block pair -> query (forward)
    size_t shift = 0, kmax = 0, oacc = 0, lacc = 0, flags = 0;   // forward
    size_t dsum = 0, dqacc = 0, dkacc = 0, dvacc = 0;   // backward
    size_t pooled = 0, part = 0;                        // decode
    size_t bmass = 0, zsel = 0, jsel = 0, dz = 0;       // proxy-head gradient (per pair-list entry)
    size_t total = 0;
};
WsLayout ws_layout(const Problem& p, int which);

// Tensor map for a bf16 tensor [e3][e2][e1][e0] with a {box0, 1, box2, 1}
// box and 128-byte swizzle.  Returns false if the driver refused it.
bool make_tmap_bf16_4d(CUtensorMap* map, const void* base, uint64_t e0, uint64_t e1, uint64_t e2,
                       uint64_t e3, uint32_t box0, uint32_t box2);

// Pairs of KV blocks (2p, 2p+1) of a sequence of nblk blocks.
inline int pair_count(int nblk) { return (nblk + 1) / 2; }

// Query blocks per work-item range of the Main Branch kernels.  The query-side
// rows one range touches (fp32 accumulators and gathered bf16 inputs of a
// group) stay near 48 MB, inside L2; larger ranges mean fewer, longer work
// items (less per-item setup).  At least four ranges per sequence keep the
// items numerous enough to balance across the SMs on shorter sequences.
inline int range_blocks(const Problem& p)
{
    const long bytes_per_block = 128L * p.G * p.d * (4 + 2);
    long rb = (48L << 20) / bytes_per_block;
    const long quarter = (p.nblk - p.qb0 + 3) / 4;
    if (rb > quarter) rb = quarter;
    if (rb < 1) rb = 1;
    if (rb > p.nblk) rb = p.nblk;
    return (int)rb;
}

// ---- tracing: CUDA events recorded around the main kernels ---------------
enum TraceKernel : int { kTraceProxy = 0, kTraceFwdMain = 1, kTraceBwdMain = 2, kTraceCount = 3 };
struct TraceEvents {
    cudaEvent_t start[kTraceCount] = {nullptr, nullptr, nullptr};
    cudaEvent_t stop[kTraceCount] = {nullptr, nullptr, nullptr};
};
TraceEvents& trace_events();   // per host thread
// Decode: splits of a row's selected blocks (one attention CTA each) and the
// launch of the four decode kernels.
int decode_splits(const Problem& p);
cudaError_t launch_decode(const Problem& pr, const int32_t* lens, const void* q, const void* qp, const void* k,
                          const void* v, const void* kp, int32_t* idx, int32_t* nsel, void* o, float* lse,
                          void* ws, const WsLayout& L, cudaStream_t st);

// Host-side count of kernel launches (msa_kernel_launches).
void count_launches(unsigned n);

inline void trace_begin(int k, cudaStream_t st)
{
    TraceEvents& t = trace_events();
    if (t.start[k]) cudaEventRecord(t.start[k], st);
}
inline void trace_end(int k, cudaStream_t st)
{
    TraceEvents& t = trace_events();
    if (t.stop[k]) cudaEventRecord(t.stop[k], st);
}

// ---- launchers (return cudaGetLastError() of their launches) -------------
cudaError_t launch_proxy_select(const Problem& p, const CUtensorMap& tm_qp, const CUtensorMap& tm_kp,
                                int32_t* idx, int32_t* nsel, float* pooled, uint32_t* status,
                                cudaStream_t st);

cudaError_t launch_block_index(const Problem& p, const int32_t* idx, const int32_t* nsel, void* ws,
                               const WsLayout& L, cudaStream_t st);

// bmass (nullable): per pair-list entry, each selected block's weight sum per head
cudaError_t launch_fwd(const Problem& p, const void* q, const void* k, const void* v,
                       const CUtensorMap& tm_k, const CUtensorMap& tm_v, const int32_t* idx,
                       const int32_t* nsel, void* o, float* lse, void* ws, const WsLayout& L,
                       float* bmass, cudaStream_t st);

// Proxy-head gradient from the pair index and block masses a forward left in ws.
cudaError_t launch_proxy_bwd(const Problem& p, const CUtensorMap& tm_kp, const void* qp, const void* kp,
                             const int32_t* idx, const int32_t* nsel, float* dqp, float* dkp, float* loss,
                             void* ws, const WsLayout& L, cudaStream_t st);

// dkv_f32: dk, dv are fp32 and receive the unrounded sums
cudaError_t launch_bwd(const Problem& p, const void* q, const void* dout, const CUtensorMap& tm_k,
                       const CUtensorMap& tm_v, const void* o, const float* lse, void* dq, void* dk,
                       void* dv, bool dkv_f32, void* ws, const WsLayout& L, cudaStream_t st);

// dst = bf16(src), n elements (a multiple of 8)
cudaError_t launch_f32_to_bf16(const float* src, void* dst, int64_t n, cudaStream_t st);

cudaError_t launch_diag_umma(int mode, int N, int K, const void* A, const void* B, float* D,
                             uint32_t* status, cudaStream_t st);
cudaError_t launch_diag_wait(uint64_t limit_ns, uint32_t* status, cudaStream_t st);

}  // namespace msa
