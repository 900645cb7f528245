// deltanet_fwd_noalloc: the forward pass for callers that cannot allocate
// device memory.
//
// Who needs this: code that runs where cudaMalloc is not allowed or not
// wanted, e.g. a host callback or plugin that must not call into the
// allocator, a CUDA-graph-based runtime that forbids allocation while it
// records, or a memory-capped process whose allocator is owned by someone
// else.  deltanet_fwd caches a per-stream workspace that it may grow with
// cudaMallocAsync; this entry point never allocates.  Its only scratch (the
// per-chunk factors T and P, and an error word) lives in one fixed-size
// __device__ array below, which every GPU that loads the library holds until
// the process exits.
//
// Scope: dense batches (no cu_seqlens), bf16, d_k = d_v = 128, chunk 64, and at
// most kNoAllocMaxUnits (chunk, head) pairs per call (B * ceil(T / 64) * H).
// Each (sequence, head) chain runs as one run of chunks (no split across SMs).
// Larger problems are rejected with DN_ERR_WORKSPACE.
//
// The first call on each device looks up the array's device address with
// cudaGetSymbolAddress (with that device current) and sets kernel attributes;
// make that first call before any stream capture.  All calls share the one
// array and it keeps the last call's contents: calls that overlap on the GPU
// (on different streams, or on different host threads) race on it.
//
// Device-side errors (a bounded wait that gave up) go to the error word at the
// head of the array.  deltanet_get_error(stream) reads and clears it, after
// synchronising `stream`: pass the stream of the no-alloc call.  Each call
// clears the word when it starts.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>

#include "../../include/deltanet.h"
#include "dn_common.cuh"
#include "dn_prep.cuh"
#include "dn_tc.cuh"

// From deltanet.cu: this host thread's bounded-wait settings (deltanet_test_set_wait).
__attribute__((visibility("hidden"))) void dn_wait_settings(unsigned long long* wait_ns, int* stall_chunk);

namespace {

constexpr int kNoAllocMaxUnits = 3072;                 // (chunk, head) pairs
constexpr size_t kNoAllocFlagBytes = 256;              // error word + padding
constexpr size_t kNoAllocScratchBytes = kNoAllocFlagBytes + (size_t)kNoAllocMaxUnits * dn::kUnitBytes;  // 48 MiB + 256 B

// In host code this name is only a host-side stand-in for the device array;
// kernels receive the address returned by cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_na_mu;
std::map<int, unsigned char*> g_na_scratch;  // device -> address of g_noalloc_scratch

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn na_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

bool na_map(CUtensorMap* m, const void* base, int64_t B, int64_t T, int64_t H, const int64_t* st) {
    std::memset(m, 0, sizeof *m);
    EncodeTiledFn enc = na_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)st[2] * 2, (cuuint64_t)st[1] * 2, (cuuint64_t)st[0] * 2};
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Once per device, with that device current: the array's device address and
// the kernels' shared-memory limits.
dn_status na_setup(int dev, unsigned char** scratch) {
    std::lock_guard<std::mutex> lk(g_na_mu);
    auto it = g_na_scratch.find(dev);
    if (it != g_na_scratch.end()) {
        *scratch = it->second;
        return DN_OK;
    }
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return DN_ERR_CUDA;
    if (cudaFuncSetAttribute(dn::tc::k_tc_chain<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dn::tc::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(dn::k_ut_prep<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dn::PrepSmem::TOTAL) != cudaSuccess ||
        cudaFuncSetAttribute(dn::k_ut_prep<false>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return DN_ERR_CUDA;
    g_na_scratch[dev] = static_cast<unsigned char*>(ptr);
    *scratch = static_cast<unsigned char*>(ptr);
    return DN_OK;
}

bool na_token_ok(const dn_tensor* t, int64_t B, int64_t T, int64_t H) {
    if (!t || t->ndim != 4 || t->dtype != DN_BF16 || t->shape[0] != B || t->shape[1] != T ||
        t->shape[2] != H || t->shape[3] != 128 || t->stride[3] != 1)
        return false;
    if ((reinterpret_cast<uintptr_t>(t->data) & 15) || !t->data) return false;
    for (int i = 0; i < 3; ++i)
        if (t->stride[i] <= 0 || (t->stride[i] * 2) % 16) return false;
    return true;
}

// Byte span [lo, hi) of a strided view (non-negative strides), and the overlap test
// deltanet_fwd applies to its outputs against its inputs and each other.
void na_span(const dn_tensor* t, uintptr_t& lo, uintptr_t& hi) {
    lo = hi = 0;
    if (!t || !t->data) return;
    int64_t last = 0;
    for (int i = 0; i < t->ndim; ++i) {
        if (t->shape[i] == 0) return;
        last += (t->shape[i] - 1) * t->stride[i];
    }
    const int64_t es = t->dtype == DN_BF16 ? 2 : 4;
    lo = reinterpret_cast<uintptr_t>(t->data);
    hi = lo + static_cast<uintptr_t>((last + 1) * es);
}
bool na_overlap(const dn_tensor* a, const dn_tensor* b) {
    uintptr_t a0, a1, b0, b1;
    na_span(a, a0, a1);
    na_span(b, b0, b1);
    if (a0 == a1 || b0 == b1) return false;
    return a0 < b1 && b0 < a1;
}

bool na_state_ok(const dn_tensor* t, int64_t N, int64_t H) {
    if (!t) return true;
    return t->ndim == 4 && t->dtype == DN_F32 && t->shape[0] == N && t->shape[1] == H &&
           t->shape[2] == 128 && t->shape[3] == 128 && t->stride[3] == 1 && t->stride[2] == 128 &&
           t->data && !(reinterpret_cast<uintptr_t>(t->data) & 15) && t->stride[0] >= 0 &&
           t->stride[1] >= 0 && !((t->stride[0] * 4) % 16) && !((t->stride[1] * 4) % 16);
}

}  // namespace

extern "C" dn_status deltanet_fwd_noalloc(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                                          const dn_tensor* beta, const dn_tensor* initial_state,
                                          int chunk_size, dn_tensor* out, dn_tensor* final_state,
                                          void* stream_ptr) {
    if (!q || !k || !v || !beta || !out || q->ndim != 4) return DN_ERR_INVALID_ARG;
    const int64_t B = q->shape[0], T = q->shape[1], H = q->shape[2];
    if (B < 1 || T < 1 || H < 1 || B * T >= (int64_t(1) << 31)) return DN_ERR_INVALID_ARG;
    if (q->dtype != DN_BF16 || q->shape[3] != 128 || v->ndim != 4 || v->shape[3] != 128)
        return DN_ERR_UNSUPPORTED;
    if (chunk_size != dn::kChunk) return DN_ERR_UNSUPPORTED;
    if (!na_token_ok(q, B, T, H) || !na_token_ok(k, B, T, H) || !na_token_ok(v, B, T, H) ||
        !na_token_ok(out, B, T, H))
        return DN_ERR_INVALID_ARG;
    if (beta->ndim != 3 || beta->dtype != DN_F32 || beta->shape[0] != B || beta->shape[1] != T ||
        beta->shape[2] != H || !beta->data || beta->stride[0] < 0 || beta->stride[1] < 0 ||
        beta->stride[2] < 0)
        return DN_ERR_INVALID_ARG;
    if (!na_state_ok(initial_state, B, H) || !na_state_ok(final_state, B, H)) return DN_ERR_INVALID_ARG;
    // the same aliasing rules as deltanet_fwd: no output overlaps an input or the other output
    const dn_tensor* ins[5] = {q, k, v, beta, initial_state};
    for (const dn_tensor* o : {static_cast<const dn_tensor*>(out), static_cast<const dn_tensor*>(final_state)}) {
        if (!o) continue;
        for (const dn_tensor* in : ins)
            if (in && na_overlap(o, in)) return DN_ERR_ALIAS;
    }
    if (final_state && na_overlap(out, final_state)) return DN_ERR_ALIAS;
    const int64_t n_c = (T + dn::kChunk - 1) / dn::kChunk;
    if (B * n_c * H > kNoAllocMaxUnits) return DN_ERR_WORKSPACE;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DN_ERR_CUDA;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return DN_ERR_CUDA;
    if (major != 10 || minor != 0) return DN_ERR_UNSUPPORTED;
    unsigned char* scratch = nullptr;
    dn_status st = na_setup(dev, &scratch);
    if (st != DN_OK) return st;

    dn::Params p;
    std::memset(&p, 0, sizeof p);
    p.nh = 1;
    p.q = q->data; p.k = k->data; p.v = v->data; p.o = out->data;
    p.beta = static_cast<const float*>(beta->data);
    p.s0 = initial_state ? static_cast<const float*>(initial_state->data) : nullptr;
    p.sT = final_state ? static_cast<float*>(final_state->data) : nullptr;
    p.q_sb = q->stride[0]; p.q_st = q->stride[1]; p.q_sh = q->stride[2];
    p.k_sb = k->stride[0]; p.k_st = k->stride[1]; p.k_sh = k->stride[2];
    p.v_sb = v->stride[0]; p.v_st = v->stride[1]; p.v_sh = v->stride[2];
    p.o_sb = out->stride[0]; p.o_st = out->stride[1]; p.o_sh = out->stride[2];
    p.b_sb = beta->stride[0]; p.b_st = beta->stride[1]; p.b_sh = beta->stride[2];
    if (initial_state) { p.s0_sn = initial_state->stride[0]; p.s0_sh = initial_state->stride[1]; }
    if (final_state) { p.sT_sn = final_state->stride[0]; p.sT_sh = final_state->stride[1]; }
    p.err = reinterpret_cast<int*>(scratch);
    dn_wait_settings(&p.wait_ns, &p.stall_chunk);
    p.wsT = scratch + kNoAllocFlagBytes;
    dn::Sched& sc = p.sched;
    sc.list = 0;
    sc.B = (int)B; sc.T = (int)T; sc.H = (int)H;
    sc.n_chunks = (int)n_c;
    sc.G = 1;
    sc.s = (int)n_c;

    CUtensorMap tq, tk, tv, to;
    if (!na_map(&tq, q->data, B, T, H, q->stride) || !na_map(&tk, k->data, B, T, H, k->stride) ||
        !na_map(&tv, v->data, B, T, H, v->stride) || !na_map(&to, out->data, B, T, H, out->stride))
        return DN_ERR_UNSUPPORTED;

    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    // the error word must start at zero; the T tiles are fully rewritten below
    if (cudaMemsetAsync(scratch, 0, sizeof(int), stream) != cudaSuccess) return DN_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DN_ERR_CUDA;
    const int64_t units = B * n_c * H;
    const int64_t cap = (int64_t)sms * dn::kPrepCtasPerSm;
    const int grid = (int)(units < cap ? units : cap);
    dn::k_ut_prep<false><<<grid, dn::kPrepThreads, dn::PrepSmem::TOTAL, stream>>>(tq, tk, p);
    dn::tc::k_tc_chain<false><<<(unsigned)(B * H), dn::tc::kThreadsTc, dn::tc::SMEM_BYTES, stream>>>(
        tq, tk, tv, to, to, p);
    return cudaGetLastError() == cudaSuccess ? DN_OK : DN_ERR_CUDA;
}

#ifdef DN_TRACE
// Timeline readers for this translation unit's copies of the trace arrays.
extern "C" int dn_trace_copy_na(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, dn::tc::g_dn_trace, sizeof(dn::tc::g_dn_trace)) == cudaSuccess ? 0 : 1;
}
extern "C" int dn_trace_copy_prep_na(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, dn::g_dn_trace_prep, sizeof(dn::g_dn_trace_prep)) == cudaSuccess ? 0 : 1;
}
#endif

// For deltanet_get_error: the error word of device `dev`'s scratch, read and cleared
// (0 when the no-alloc entry point has not run on that device).  Returns nonzero on a
// CUDA error.  The caller has synchronised the stream of the call that wrote it.
__attribute__((visibility("hidden"))) int dn_noalloc_take_error(int dev, int* word) {
    *word = 0;
    unsigned char* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_na_mu);
        auto it = g_na_scratch.find(dev);
        if (it == g_na_scratch.end()) return 0;
        scratch = it->second;
    }
    int h = 0;
    if (cudaMemcpy(&h, scratch, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return 1;
    if (h != 0 && cudaMemset(scratch, 0, sizeof h) != cudaSuccess) return 1;
    *word = h;
    return 0;
}
