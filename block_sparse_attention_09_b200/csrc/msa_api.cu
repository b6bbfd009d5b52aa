// C ABI of libmsa.so: argument validation, workspace layout, tensor maps and
// the order of launches for each phase.  See include/msa.h for the contract.
#include <math.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/msa.h"
#include "msa_internal.h"

namespace msa {

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

WsLayout ws_layout(const Problem& p, int which)
{
    if (which == MSA_PROXY_BWD) {
        // the forward's layout (index, forward regions) at its own offsets,
        // then the per-entry buffers of the proxy-head gradient past anything
        // a forward or a main backward on the same workspace writes
        WsLayout L = ws_layout(p, MSA_FWD);
        const size_t bwd = ws_layout(p, MSA_BWD).total;
        size_t off = L.total > bwd ? L.total : bwd;
        auto take = [&](size_t bytes) { const size_t at = off; off = align256(off + bytes); return at; };
        const size_t E = (size_t)p.B * p.Hp * p.T * p.topk;   // pair-list entries, at most
        L.bmass = take(E * 2 * p.G * 4);
        L.zsel = take(E * 2 * 4);
        L.jsel = take(E * 2 * 4);
        L.dz = take(E * 2 * 4);
        L.total = off;
        return L;
    }
    WsLayout L;
    size_t off = 256;   // status words
    const size_t BH = (size_t)p.B * p.Hp;
    const size_t rows = (size_t)p.rows_q();
    auto take = [&](size_t bytes) { const size_t at = off; off = align256(off + bytes); return at; };
    if (which == MSA_FWD || which == MSA_BWD) {
        L.cnt = take(BH * p.nblk * p.nblk * 4);
        L.tot = take(BH * p.nblk * 4);
        L.ptr = take(BH * (p.nblk + 1) * 4);
        L.tok = take(BH * (size_t)p.T * p.topk * 4);
        const size_t np = (size_t)pair_count(p.nblk);
        L.cnt2 = take(BH * p.nblk * np * 4);
        L.tot2 = take(BH * np * 4);
        L.ptr2 = take(BH * (np + 1) * 4);
        L.tok2 = take(BH * (size_t)p.T * p.topk * 4);
    }
    if (which == MSA_FWD) {
        L.shift = take(rows * 4);
        L.kmax = take((size_t)p.B * p.Hkv * p.nblk * 4);
        L.oacc = take(rows * p.d * 4);
        L.lacc = take(rows * 4);
        L.flags = take(rows * 4);
    }
    if (which == MSA_DECODE) {
        L.pooled = take(BH * p.nblk * 4);
        L.part = take((size_t)p.B * p.Hkv * decode_splits(p) * p.G * (p.d + 2) * 4);
    }
    if (which == MSA_BWD) {
        L.dsum = take(rows * 4);
        L.dqacc = take(rows * p.d * 4);
        L.dkacc = take((size_t)p.B * p.T * p.Hkv * p.d * 4);
        L.dvacc = take((size_t)p.B * p.T * p.Hkv * p.d * 4);
    }
    L.total = off;
    return L;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)f;
    });
    return fn;
}

bool make_tmap_bf16_4d(CUtensorMap* map, const void* base, uint64_t e0, uint64_t e1, uint64_t e2, uint64_t e3,
                       uint32_t box0, uint32_t box2)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {e0, e1, e2, e3};
    const cuuint64_t strides[3] = {e0 * 2, e0 * e1 * 2, e0 * e1 * e2 * 2};   // bytes, dims 1..3
    const cuuint32_t box[4] = {box0, 1, box2, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    memset(map, 0, sizeof(*map));
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

TraceEvents& trace_events()
{
    static thread_local TraceEvents t;
    return t;
}

static std::atomic<unsigned long long> g_launches{0};

void count_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

}  // namespace msa

using namespace msa;

namespace {

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

// decode: idx holds one row per (b, group), so the full-sequence index bound
// does not apply
int to_problem(const msa_dims* d, Problem* p, bool decode = false)
{
    if (!d) return MSA_ERR_NULL_PTR;
    if (d->B < 0 || d->T < 0 || d->T > kMaxT || d->Hkv < 1 || d->Hq < 1 || d->Hq % d->Hkv != 0 ||
        d->Hp != d->Hkv || d->block != kBlock || d->topk < 1 || d->topk > kMaxTopk)
        return MSA_ERR_INVALID_DIMS;
    const int G = d->Hq / d->Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return MSA_ERR_INVALID_DIMS;
    if (d->d != 64 && d->d != 128) return MSA_ERR_INVALID_DIMS;
    if (d->dp < 8 || d->dp > 64 || d->dp % 8 != 0) return MSA_ERR_INVALID_DIMS;
    if (!isfinite(d->scale)) return MSA_ERR_INVALID_DIMS;
    if (d->window < 0 || d->window > d->topk || d->dilation < 0 || d->dilation > kMaxT) return MSA_ERR_INVALID_DIMS;
    // first computed query row: a block boundary inside [0, T]; decode has one query per sequence
    if (d->q_begin < 0 || d->q_begin % kBlock != 0 || d->q_begin > d->T || (decode && d->q_begin != 0))
        return MSA_ERR_INVALID_DIMS;
    p->B = d->B; p->T = d->T; p->Hq = d->Hq; p->Hkv = d->Hkv; p->Hp = d->Hp;
    p->d = d->d; p->dp = d->dp; p->topk = d->topk;
    p->nblk = (d->T + kBlock - 1) / kBlock;
    p->window = d->window > 0 ? d->window : 1;
    p->dilation = d->dilation > 0 ? d->dilation : 1;
    p->G = G;
    p->q0 = d->q_begin;
    p->qb0 = d->q_begin / kBlock;
    p->scale = d->scale != 0.f ? d->scale : 1.0f / sqrtf((float)d->d);
    if (!decode && (int64_t)p->B * p->Hp * p->T * p->topk > (int64_t)INT32_MAX) return MSA_ERR_INVALID_DIMS;
    return MSA_OK;
}

int check_device()
{
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MSA_ERR_DEVICE;
    // bind the device's primary context to this host thread: tensor-map
    // encoding needs a current context, and a caller's worker thread (an
    // autograd engine thread, say) may not have one yet
    if (cudaSetDevice(dev) != cudaSuccess) return MSA_ERR_DEVICE;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MSA_ERR_DEVICE;
    return major == 10 ? MSA_OK : MSA_ERR_DEVICE;
}

int check_ws(const Problem& p, int which, void* ws, size_t ws_bytes, WsLayout* L)
{
    *L = ws_layout(p, which);
    if (!ws) return MSA_ERR_NULL_PTR;
    if (!aligned(ws, 256)) return MSA_ERR_MISALIGNED;
    if (ws_bytes < L->total) return MSA_ERR_WS_TOO_SMALL;
    return MSA_OK;
}

bool empty(const Problem& p) { return p.B == 0 || p.T == 0 || p.q0 >= p.T; }

// A shard with no query row (q_begin == T, with B and T > 0) enqueues no
// kernel, but it still clears the workspace's status words, so that
// msa_check_status and msa_fallback_rows describe this call and not an
// earlier one.
bool no_rows(const Problem& p) { return p.B > 0 && p.T > 0 && p.q0 >= p.T; }
int clear_status(void* ws, const WsLayout& L, void* stream)
{
    int rc;
    if ((rc = check_device()) != MSA_OK) return rc;
    if (cudaMemsetAsync((uint8_t*)ws + L.status, 0, 256, (cudaStream_t)stream) != cudaSuccess) return MSA_ERR_LAUNCH;
    return MSA_OK;
}

}  // namespace

extern "C" {

size_t msa_workspace_size(const msa_dims* dims, int which)
{
    Problem p;
    if (to_problem(dims, &p, which == MSA_DECODE) != MSA_OK) return 0;
    if (which < MSA_SELECT || which > MSA_PROXY_BWD) return 0;
    return ws_layout(p, which).total;
}

int msa_proxy_select(const msa_dims* dims, const void* qp, const void* kp, int32_t* idx, int32_t* nsel,
                     float* pooled_dbg, void* ws, size_t ws_bytes, void* stream)
{
    Problem p;
    int rc = to_problem(dims, &p);
    if (rc != MSA_OK) return rc;
    WsLayout L;
    if ((rc = check_ws(p, MSA_SELECT, ws, ws_bytes, &L)) != MSA_OK) return rc;
    if (no_rows(p)) return clear_status(ws, L, stream);
    if (empty(p)) return MSA_OK;
    if (!qp || !kp || !idx || !nsel) return MSA_ERR_NULL_PTR;
    if (!aligned(qp, 16) || !aligned(kp, 16) || !aligned(idx, 16) || !aligned(nsel, 16) ||
        (pooled_dbg && !aligned(pooled_dbg, 16)))
        return MSA_ERR_MISALIGNED;
    if ((rc = check_device()) != MSA_OK) return rc;
    CUtensorMap tq, tk;
    // query tiles of 128 rows; key tiles of 256 rows (two key blocks per MMA)
    if (!make_tmap_bf16_4d(&tq, qp, p.dp, p.Hp, p.T, p.B, 64, 128) ||
        !make_tmap_bf16_4d(&tk, kp, p.dp, p.Hp, p.T, p.B, 64, 256))
        return MSA_ERR_DRIVER;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t* status = (uint32_t*)((uint8_t*)ws + L.status);
    if (cudaMemsetAsync(status, 0, 256, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    if (launch_proxy_select(p, tq, tk, idx, nsel, pooled_dbg, status, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    return MSA_OK;
}

int msa_fwd_ex(const msa_dims* dims, const void* q, const void* k, const void* v, const int32_t* idx,
               const int32_t* nsel, void* o, float* lse, void* ws, size_t ws_bytes, void* stream, int flags)
{
    Problem p;
    int rc = to_problem(dims, &p);
    if (rc != MSA_OK) return rc;
    WsLayout L;
    const bool mass = (flags & MSA_BLOCK_MASS) != 0;
    if ((rc = check_ws(p, mass ? MSA_PROXY_BWD : MSA_FWD, ws, ws_bytes, &L)) != MSA_OK) return rc;
    if (no_rows(p)) return clear_status(ws, L, stream);
    if (empty(p)) return MSA_OK;
    if (!q || !k || !v || !idx || !nsel || !o || !lse) return MSA_ERR_NULL_PTR;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(idx, 16) || !aligned(nsel, 16) ||
        !aligned(o, 16) || !aligned(lse, 16))
        return MSA_ERR_MISALIGNED;
    if ((rc = check_device()) != MSA_OK) return rc;
    CUtensorMap tk, tv;
    if (!make_tmap_bf16_4d(&tk, k, p.d, p.Hkv, p.T, p.B, 64, 128) ||
        !make_tmap_bf16_4d(&tv, v, p.d, p.Hkv, p.T, p.B, 64, 128))
        return MSA_ERR_DRIVER;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t* status = (uint32_t*)((uint8_t*)ws + L.status);
    if (cudaMemsetAsync(status, 0, 256, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    if (!(flags & MSA_REUSE_INDEX) && launch_block_index(p, idx, nsel, ws, L, st) != cudaSuccess)
        return MSA_ERR_LAUNCH;
    float* bmass = mass ? (float*)((uint8_t*)ws + L.bmass) : nullptr;
    if (launch_fwd(p, q, k, v, tk, tv, idx, nsel, o, lse, ws, L, bmass, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    return MSA_OK;
}

int msa_fwd(const msa_dims* dims, const void* q, const void* k, const void* v, const int32_t* idx,
            const int32_t* nsel, void* o, float* lse, void* ws, size_t ws_bytes, void* stream)
{
    return msa_fwd_ex(dims, q, k, v, idx, nsel, o, lse, ws, ws_bytes, stream, 0);
}

int msa_bwd_ex(const msa_dims* dims, const void* q, const void* k, const void* v, const void* o,
               const void* dout, const float* lse, const int32_t* idx, const int32_t* nsel, void* dq, void* dk,
               void* dv, void* ws, size_t ws_bytes, void* stream, int flags)
{
    Problem p;
    int rc = to_problem(dims, &p);
    if (rc != MSA_OK) return rc;
    WsLayout L;
    if ((rc = check_ws(p, MSA_BWD, ws, ws_bytes, &L)) != MSA_OK) return rc;
    if (p.B > 0 && p.T > 0 && p.q0 >= p.T) {
        // no query row computed: the partial dK, dV are zero
        if (!dk || !dv) return MSA_ERR_NULL_PTR;
        if ((rc = clear_status(ws, L, stream)) != MSA_OK) return rc;
        const size_t bytes = (size_t)p.B * p.T * p.Hkv * p.d * ((flags & MSA_DKV_F32) ? 4 : 2);
        if (cudaMemsetAsync(dk, 0, bytes, (cudaStream_t)stream) != cudaSuccess ||
            cudaMemsetAsync(dv, 0, bytes, (cudaStream_t)stream) != cudaSuccess)
            return MSA_ERR_LAUNCH;
        return MSA_OK;
    }
    if (empty(p)) return MSA_OK;
    if (!q || !k || !v || !o || !dout || !lse || !idx || !nsel || !dq || !dk || !dv) return MSA_ERR_NULL_PTR;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
        !aligned(lse, 16) || !aligned(idx, 16) || !aligned(nsel, 16) || !aligned(dq, 16) || !aligned(dk, 16) ||
        !aligned(dv, 16))
        return MSA_ERR_MISALIGNED;
    if ((rc = check_device()) != MSA_OK) return rc;
    CUtensorMap tk, tv;
    if (!make_tmap_bf16_4d(&tk, k, p.d, p.Hkv, p.T, p.B, 64, 128) ||
        !make_tmap_bf16_4d(&tv, v, p.d, p.Hkv, p.T, p.B, 64, 128))
        return MSA_ERR_DRIVER;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t* status = (uint32_t*)((uint8_t*)ws + L.status);
    if (cudaMemsetAsync(status, 0, 256, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    if (!(flags & MSA_REUSE_INDEX) && launch_block_index(p, idx, nsel, ws, L, st) != cudaSuccess)
        return MSA_ERR_LAUNCH;
    if (launch_bwd(p, q, dout, tk, tv, o, lse, dq, dk, dv, (flags & MSA_DKV_F32) != 0, ws, L, st) != cudaSuccess)
        return MSA_ERR_LAUNCH;
    return MSA_OK;
}

int msa_bwd(const msa_dims* dims, const void* q, const void* k, const void* v, const void* o, const void* dout,
            const float* lse, const int32_t* idx, const int32_t* nsel, void* dq, void* dk, void* dv, void* ws,
            size_t ws_bytes, void* stream)
{
    return msa_bwd_ex(dims, q, k, v, o, dout, lse, idx, nsel, dq, dk, dv, ws, ws_bytes, stream, 0);
}

int msa_decode(const msa_dims* dims, const int32_t* lens, const void* q, const void* qp, const void* k,
               const void* v, const void* kp, int32_t* idx, int32_t* nsel, void* o, float* lse, void* ws,
               size_t ws_bytes, void* stream)
{
    Problem p;
    int rc = to_problem(dims, &p, true);
    if (rc != MSA_OK) return rc;
    WsLayout L;
    if ((rc = check_ws(p, MSA_DECODE, ws, ws_bytes, &L)) != MSA_OK) return rc;
    if (empty(p)) return MSA_OK;
    if (!q || !qp || !k || !v || !kp || !idx || !nsel || !o || !lse) return MSA_ERR_NULL_PTR;
    if (!aligned(q, 16) || !aligned(qp, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(kp, 16) ||
        !aligned(idx, 4) || !aligned(nsel, 4) || !aligned(o, 16) || !aligned(lse, 4) || (lens && !aligned(lens, 4)))
        return MSA_ERR_MISALIGNED;
    if ((rc = check_device()) != MSA_OK) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t* status = (uint32_t*)((uint8_t*)ws + L.status);
    if (cudaMemsetAsync(status, 0, 256, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    if (launch_decode(p, lens, q, qp, k, v, kp, idx, nsel, o, lse, ws, L, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    return MSA_OK;
}

int msa_proxy_bwd(const msa_dims* dims, const void* qp, const void* kp, const int32_t* idx, const int32_t* nsel,
                  float* dqp, float* dkp, float* loss, void* ws, size_t ws_bytes, void* stream)
{
    Problem p;
    int rc = to_problem(dims, &p);
    if (rc != MSA_OK) return rc;
    WsLayout L;
    if ((rc = check_ws(p, MSA_PROXY_BWD, ws, ws_bytes, &L)) != MSA_OK) return rc;
    if (no_rows(p)) {   // no query row: dkp is zero everywhere
        if (!dkp) return MSA_ERR_NULL_PTR;
        if ((rc = clear_status(ws, L, stream)) != MSA_OK) return rc;
        if (cudaMemsetAsync(dkp, 0, sizeof(float) * (size_t)p.B * p.T * p.Hp * p.dp, (cudaStream_t)stream) !=
            cudaSuccess)
            return MSA_ERR_LAUNCH;
        return MSA_OK;
    }
    if (empty(p)) return MSA_OK;
    if (!qp || !kp || !idx || !nsel || !dqp || !dkp || !loss) return MSA_ERR_NULL_PTR;
    if (!aligned(qp, 16) || !aligned(kp, 16) || !aligned(idx, 16) || !aligned(nsel, 16) || !aligned(dqp, 16) ||
        !aligned(dkp, 16) || !aligned(loss, 16))
        return MSA_ERR_MISALIGNED;
    if ((rc = check_device()) != MSA_OK) return rc;
    CUtensorMap tk;
    if (!make_tmap_bf16_4d(&tk, kp, p.dp, p.Hp, p.T, p.B, 64, 256)) return MSA_ERR_DRIVER;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t* status = (uint32_t*)((uint8_t*)ws + L.status);
    if (cudaMemsetAsync(status, 0, 256, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    if (launch_proxy_bwd(p, tk, qp, kp, idx, nsel, dqp, dkp, loss, ws, L, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    return MSA_OK;
}

int msa_f32_to_bf16(const float* src, void* dst, int64_t n, void* stream)
{
    if (n < 0 || n % 8 != 0) return MSA_ERR_INVALID_DIMS;
    if (n == 0) return MSA_OK;
    if (!src || !dst) return MSA_ERR_NULL_PTR;
    if (!aligned(src, 16) || !aligned(dst, 16)) return MSA_ERR_MISALIGNED;
    int rc = check_device();
    if (rc != MSA_OK) return rc;
    return launch_f32_to_bf16(src, dst, n, (cudaStream_t)stream) == cudaSuccess ? MSA_OK : MSA_ERR_LAUNCH;
}

int msa_check_status(const void* ws, void* stream, uint32_t* code)
{
    if (!ws) return MSA_ERR_NULL_PTR;
    uint32_t words[2] = {0, 0};
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MSA_ERR_LAUNCH;
    if (cudaMemcpy(words, ws, sizeof(words), cudaMemcpyDeviceToHost) != cudaSuccess) return MSA_ERR_LAUNCH;
    if (code) *code = words[0] ? words[0] : (words[1] ? kStIndexError : 0u);
    if (words[0]) return MSA_ERR_TIMEOUT;
    if (words[1]) return MSA_ERR_INDEX;
    return MSA_OK;
}

int msa_fallback_rows(const void* ws, void* stream, int64_t* rows)
{
    if (!ws || !rows) return MSA_ERR_NULL_PTR;
    uint32_t w = 0;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MSA_ERR_LAUNCH;
    if (cudaMemcpy(&w, (const uint32_t*)ws + 2, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MSA_ERR_LAUNCH;
    *rows = (int64_t)w;
    return MSA_OK;
}

const char* msa_strerror(int s)
{
    switch (s) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_DIMS: return "invalid dimensions";
    case MSA_ERR_NULL_PTR: return "null pointer";
    case MSA_ERR_MISALIGNED: return "misaligned pointer";
    case MSA_ERR_WS_TOO_SMALL: return "workspace too small";
    case MSA_ERR_LAUNCH: return "CUDA launch failed";
    case MSA_ERR_TIMEOUT: return "device wait timed out";
    case MSA_ERR_DEVICE: return "device is not sm_100";
    case MSA_ERR_DRIVER: return "tensor map encoding failed";
    case MSA_ERR_INDEX: return "block index out of range";
    default: return "unknown status";
    }
}

uint64_t msa_kernel_launches(void) { return (uint64_t)msa::g_launches.load(std::memory_order_relaxed); }

int msa_set_kernel_events(int kernel, void* start, void* stop)
{
    if (kernel < 0 || kernel >= kTraceCount) return MSA_ERR_INVALID_DIMS;
    TraceEvents& t = trace_events();
    t.start[kernel] = (cudaEvent_t)start;
    t.stop[kernel] = (cudaEvent_t)stop;
    return MSA_OK;
}

int msa_diag_umma(int mode, int N, int K, const void* A, const void* B, float* D, void* ws, void* stream)
{
    if (mode < 0 || mode > 4 || (N != 64 && N != 128) || (K != 64 && K != 128)) return MSA_ERR_INVALID_DIMS;
    if (!A || !B || !D || !ws) return MSA_ERR_NULL_PTR;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || !aligned(ws, 256)) return MSA_ERR_MISALIGNED;
    int rc = check_device();
    if (rc != MSA_OK) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(ws, 0, 256, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    if (launch_diag_umma(mode, N, K, A, B, D, (uint32_t*)ws, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    return msa_check_status(ws, stream, nullptr);
}

int msa_diag_wait_timeout(uint64_t limit_ns, void* ws, void* stream)
{
    if (!ws) return MSA_ERR_NULL_PTR;
    if (!aligned(ws, 256)) return MSA_ERR_MISALIGNED;
    int rc = check_device();
    if (rc != MSA_OK) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(ws, 0, 256, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    if (launch_diag_wait(limit_ns, (uint32_t*)ws, st) != cudaSuccess) return MSA_ERR_LAUNCH;
    return msa_check_status(ws, stream, nullptr);
}

}  // extern "C"
