// Host side of the C ABI declared in include/deltanet.h: argument checks,
// per-stream workspace, scheduling and kernel launches.  No computation of the
// method happens on the host.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <type_traits>
#include <utility>

#include "../../include/deltanet.h"
#include "dn_chain.cuh"
#include "dn_common.cuh"
#include "dn_prep.cuh"
#include "dn_sched.cuh"
#include "dn_tc.cuh"
#include "dn_tc_sum.cuh"

using namespace dn;

// Shared with deltanet_noalloc.cu (not exported): this thread's bounded-wait settings
// for the next calls, and the no-alloc scratch's error word of a device (read and
// cleared; 0 when that entry point never ran on the device).
__attribute__((visibility("hidden"))) void dn_wait_settings(unsigned long long* wait_ns, int* stall_chunk);
__attribute__((visibility("hidden"))) int dn_noalloc_take_error(int dev, int* word);

namespace {

thread_local int g_last_G = 0, g_last_s = 0, g_last_s0 = 0, g_last_launches = 0;
// deltanet_test_set_wait: time-out of the bounded device waits (0: 2 s) and the test stall
thread_local unsigned long long g_wait_ns = 0;
thread_local int g_stall_chunk = 0;
thread_local cudaEvent_t g_ev_start = nullptr, g_ev_stop = nullptr;

struct StreamWs {
    int* flag = nullptr;  // [0] error flag
    char* buf = nullptr;
    size_t cap = 0;
};

std::mutex g_mu;
std::map<std::pair<int, cudaStream_t>, StreamWs> g_ws;
std::set<std::pair<int, const void*>> g_attr_done;
std::map<int, int> g_dev_ok;     // device -> 1 ok, 0 unsupported
std::map<int, int> g_dev_sms;

int64_t elem_size(int32_t dt) { return dt == DN_F32 ? 4 : dt == DN_BF16 ? 2 : dt == DN_I32 ? 4 : 0; }

bool shape_eq(const dn_tensor* t, int ndim, const int64_t* dims) {
    if (!t || t->ndim != ndim) return false;
    for (int i = 0; i < ndim; ++i)
        if (t->shape[i] != dims[i]) return false;
    return true;
}

int64_t numel(const dn_tensor* t) {
    int64_t n = 1;
    for (int i = 0; i < t->ndim; ++i) n *= t->shape[i];
    return n;
}

// Byte span [lo, hi) touched by a strided view (non-negative strides only).
bool span(const dn_tensor* t, uintptr_t& lo, uintptr_t& hi) {
    lo = hi = 0;
    if (!t || numel(t) == 0) return true;
    int64_t last = 0;
    for (int i = 0; i < t->ndim; ++i) {
        if (t->stride[i] < 0) return false;
        last += (t->shape[i] - 1) * t->stride[i];
    }
    const int64_t es = elem_size(t->dtype);
    lo = reinterpret_cast<uintptr_t>(t->data);
    hi = lo + static_cast<uintptr_t>((last + 1) * es);
    return true;
}

bool overlap(const dn_tensor* a, const dn_tensor* b) {
    uintptr_t a0, a1, b0, b1;
    span(a, a0, a1);
    span(b, b0, b1);
    if (a0 == a1 || b0 == b1) return false;
    return a0 < b1 && b0 < a1;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// q/k/v/out: [B, T, H, d], stride[3] == 1, 16-byte aligned rows and strides.
bool token_tensor_ok(const dn_tensor* t) {
    if (t->stride[3] != 1) return false;
    const int64_t es = elem_size(t->dtype);
    if (numel(t) == 0) return true;
    if (!t->data || !aligned16(t->data)) return false;
    for (int i = 0; i < 3; ++i)
        if (t->stride[i] < 0 || (t->stride[i] * es) % 16 != 0) return false;
    return true;
}

bool state_tensor_ok(const dn_tensor* t, int64_t dv) {
    if (t->dtype != DN_F32 || t->stride[3] != 1 || t->stride[2] != dv) return false;
    if (numel(t) == 0) return true;
    if (!t->data || !aligned16(t->data)) return false;
    return t->stride[0] >= 0 && t->stride[1] >= 0 && (t->stride[0] * 4) % 16 == 0 &&
           (t->stride[1] * 4) % 16 == 0;
}

dn_status device_check(int& dev, int& sms) {
    if (cudaGetDevice(&dev) != cudaSuccess) return DN_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_dev_ok.find(dev);
    if (it == g_dev_ok.end()) {
        int major = 0, minor = 0, n = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return DN_ERR_CUDA;
        g_dev_ok[dev] = (major == 10 && minor == 0) ? 1 : 0;
        g_dev_sms[dev] = n;
        it = g_dev_ok.find(dev);
    }
    sms = g_dev_sms[dev];
    return it->second ? DN_OK : DN_ERR_UNSUPPORTED;
}

template <typename K>
dn_status set_smem(K* kernel, int dev, int bytes) {
    std::lock_guard<std::mutex> lk(g_mu);
    auto key = std::make_pair(dev, reinterpret_cast<const void*>(kernel));
    if (g_attr_done.count(key)) return DN_OK;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
        return DN_ERR_CUDA;
    g_attr_done.insert(key);
    return DN_OK;
}

// Workspace of `bytes` for (dev, stream); grows stream-ordered.
dn_status get_ws(int dev, cudaStream_t stream, size_t bytes, StreamWs& out) {
    std::lock_guard<std::mutex> lk(g_mu);
    StreamWs& w = g_ws[std::make_pair(dev, stream)];
    if (!w.flag) {
        if (cudaMalloc(&w.flag, 256) != cudaSuccess) {
            w.flag = nullptr;
            return DN_ERR_WORKSPACE;
        }
        if (cudaMemset(w.flag, 0, 256) != cudaSuccess) return DN_ERR_CUDA;
    }
    if (bytes > w.cap) {
        if (w.buf) cudaFreeAsync(w.buf, stream);
        w.buf = nullptr;
        w.cap = 0;
        size_t want = std::max(bytes, (size_t)1 << 20);
        if (cudaMallocAsync(reinterpret_cast<void**>(&w.buf), want, stream) != cudaSuccess) {
            w.buf = nullptr;
            return DN_ERR_WORKSPACE;
        }
        w.cap = want;
    }
    out = w;
    return DN_OK;
}

// A second stream (and a fork / join event pair) per (device, caller's stream), for
// work that runs next to the caller's stream within one call.
struct AuxStream {
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
std::map<std::pair<int, cudaStream_t>, AuxStream> g_aux;

dn_status get_aux(int dev, cudaStream_t stream, AuxStream& out) {
    std::lock_guard<std::mutex> lk(g_mu);
    AuxStream& a = g_aux[std::make_pair(dev, stream)];
    if (!a.stream) {
        if (cudaStreamCreateWithFlags(&a.stream, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&a.join, cudaEventDisableTiming) != cudaSuccess) {
            a = AuxStream();
            return DN_ERR_CUDA;
        }
    }
    out = a;
    return DN_OK;
}

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// TMA map of a bf16 [B, T, H, 128] tensor (element strides sb, st, sh): boxes of
// 64 tokens x 64 channels of one head, 128-byte swizzle, zero fill past T.
dn_status make_token_map(CUtensorMap* m, const void* base, int64_t B, int64_t T, int64_t H,
                         int64_t sb, int64_t st, int64_t sh, int rows = 64) {
    std::memset(m, 0, sizeof *m);
    if (B * T == 0) return DN_OK;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return DN_ERR_CUDA;
    cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)sh * 2, (cuuint64_t)st * 2, (cuuint64_t)(sb > 0 ? sb : T * st) * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DN_OK : DN_ERR_UNSUPPORTED;
}

// 2-D map over the segment transition products P_g (rows of DK fp32), boxes of
// 32 columns x DK rows with the 128-byte swizzle (the segment scan's operand layout).
dn_status make_p_map(CUtensorMap* m, const void* base, int64_t rows, int dk) {
    std::memset(m, 0, sizeof *m);
    if (rows == 0) return DN_OK;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return DN_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)dk, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)dk * 4};
    cuuint32_t box[2] = {32, (cuuint32_t)dk};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DN_OK : DN_ERR_UNSUPPORTED;
}

struct Dims {
    int64_t B, T, H, dk, dv, N;
    bool varlen;
};

template <typename E, int DK, int DV, int STAGES, bool GATED, bool KDA = false>
dn_status launch(Params p, const Dims& d, int dev, int sms, cudaStream_t stream, int forced_s,
                 const int* cu) {
    // bf16 DeltaNet, Gated DeltaNet and the Gated Delta Product with d_k = d_v = 128 run on
    // the tensor-core (tcgen05) kernels (with or without the chunk-start states), the other
    // shapes on the mma.sync chain kernels.  Kimi Delta Attention (a decay per key channel)
    // with d_k = d_v = 128 runs on its tensor-core pre-pass and boundary kernel when a dense
    // batch's chains are not split (one run per chain; there is no KDA summary pass on the
    // tensor cores), otherwise on the mma.sync chain kernels.
    constexpr bool kBf16x128 = std::is_same<E, __nv_bfloat16>::value && DK == 128 && DV == 128;
    constexpr bool kTcShape = !KDA && kBf16x128;
    bool use_tc = kTcShape && (p.nh <= 1 || GATED);
    if constexpr (KDA && kBf16x128) {
        if (!d.varlen) {
            const int64_t n_c = (d.T + kChunk - 1) / kChunk;
            const int s1 = forced_s > 0 ? (forced_s & 0xffff)
                                        : choose_dense(CostModel{}, (int)(d.N * d.H), (int)n_c, sms,
                                                       kAutoMaxSlots, false).s;
            use_tc = s1 >= n_c;
        }
    }
    using LC = ChainSmem<E, DK, DV, true, true, STAGES, GATED, KDA>;
    using LH = ChainSmem<E, DK, DV, true, false, STAGES, GATED, KDA>;
    using LP = ChainSmem<E, DK, DK, false, false, STAGES, GATED, KDA>;
    static_assert(LC::TOTAL <= 232448 && LH::TOTAL <= 232448 && LP::TOTAL <= 232448,
                  "chain kernel shared memory");
    const int smemC = LC::TOTAL;
    const int smemA = LH::TOTAL > LP::TOTAL ? LH::TOTAL : LP::TOTAL;
    const int smemS8 = scan_smem_bytes<DK, 8>(), smemS16 = scan_smem_bytes<DK, 16>();
    auto* kC = k_boundary<E, DK, DV, STAGES, GATED, KDA>;
    auto* kA = k_summary<E, DK, DV, STAGES, GATED, KDA>;
    auto* kS8 = k_scan<DK, DV, 8>;
    auto* kS16 = k_scan<DK, DV, 16>;
    // the Gated Delta Product runs the instances that handle several steps per token
    const bool multi = GATED && p.nh > 1;
    // KDA's tensor-core instances: the gated layout with K<- and K-> from its own pre-pass
    constexpr bool kKdaTc = KDA && kBf16x128;
    auto* kCt = kKdaTc ? tc::k_tc_chain<true, false, kKdaTc>
                       : (multi ? tc::k_tc_chain<GATED, GATED> : tc::k_tc_chain<GATED, false>);
    auto* kAt = tcs::k_tc_summary<GATED>;
    auto* kPrep = multi ? k_ut_prep<GATED, GATED> : k_ut_prep<GATED, false>;
    constexpr int smemPrep = kKdaTc ? KdaPrepLay::TOTAL : PrepSmemT<GATED>::TOTAL;
    constexpr int smemCt = kKdaTc ? tc::TcLay<true, true>::SMEM_BYTES : tc::TcLay<GATED>::SMEM_BYTES;
    constexpr int smemAt = tcs::SumLay<GATED>::SMEM_BYTES;
    dn_status st;
    if (use_tc) {
        if ((st = set_smem(kCt, dev, smemCt)) != DN_OK) return st;
        if ((st = set_smem(kAt, dev, smemAt)) != DN_OK) return st;
        if constexpr (kKdaTc) {
            auto* kKp = k_kda_prep<DK>;
            if ((st = set_smem(kKp, dev, smemPrep)) != DN_OK) return st;
            if (cudaFuncSetAttribute(kKp, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     cudaSharedmemCarveoutMaxShared) != cudaSuccess)
                return DN_ERR_CUDA;
        } else {
            if ((st = set_smem(kPrep, dev, smemPrep)) != DN_OK) return st;
            // several pre-pass CTAs share an SM: ask for the largest shared-memory carveout
            if (cudaFuncSetAttribute(kPrep, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     cudaSharedmemCarveoutMaxShared) != cudaSuccess)
                return DN_ERR_CUDA;
        }
    } else {
        if ((st = set_smem(kC, dev, smemC)) != DN_OK) return st;
        if ((st = set_smem(kA, dev, smemA)) != DN_OK) return st;
    }
    if ((st = set_smem(kS8, dev, smemS8)) != DN_OK) return st;
    if ((st = set_smem(kS16, dev, smemS16)) != DN_OK) return st;
    CUtensorMap tq, tk, tv, to, toc;
    if (use_tc) {
        const int64_t Bq = d.varlen ? 1 : d.B;
        const int64_t Tq = d.T / (p.nh > 1 ? p.nh : 1);  // q and out: one row per token
        if ((st = make_token_map(&tq, p.q, Bq, Tq, d.H, p.q_sb, p.q_st, p.q_sh)) != DN_OK) return st;
        if ((st = make_token_map(&tk, p.k, Bq, d.T, d.H, p.k_sb, p.k_st, p.k_sh)) != DN_OK) return st;
        if ((st = make_token_map(&tv, p.v, Bq, d.T, d.H, p.v_sb, p.v_st, p.v_sh)) != DN_OK) return st;
        if ((st = make_token_map(&to, p.o, Bq, Tq, d.H, p.o_sb, p.o_st, p.o_sh)) != DN_OK) return st;
        // Gated Delta Product: a chunk's outputs are 64 / n_h token rows
        toc = to;
        if (p.nh > 1 && kChunk % p.nh == 0 &&
            (st = make_token_map(&toc, p.o, Bq, Tq, d.H, p.o_sb, p.o_st, p.o_sh, kChunk / p.nh)) != DN_OK)
            return st;
    }

    const int64_t n_c_max = (d.T + kChunk - 1) / kChunk;
    const int64_t chains = d.N * d.H;
    CostModel model;
    if (use_tc && !KDA) model.a = kTcSummaryCost;
    size_t bytes = 0;
    int64_t slots = 0, nC = 0, nA = 0, nScan = 0;
    int G = 1, s = 1, s0 = 0;
    bool e_in_c = false;
    if (!d.varlen) {
        if (forced_s > 0) {
            s = forced_s & 0xffff;
            s0 = (forced_s >> 16) & 0x7fff;
            if (s < 1 || s0 > s) return DN_ERR_INVALID_ARG;
        } else {
            SegChoice ch = choose_dense(model, (int)chains, (int)n_c_max, sms, kAutoMaxSlots, use_tc && !KDA);
            s = ch.s;
            s0 = ch.s0;
        }
        // run 0 has s0 chunks (s when s0 == 0), the others s
        const int64_t first = s0 > 0 ? s0 : s;
        G = n_c_max > first ? (int)(1 + (n_c_max - first + s - 1) / s) : 1;
        slots = chains * (G - 1);
        if (slots > kMaxSlots) return DN_ERR_WORKSPACE;
        nC = chains * G;
        // tensor-core path: run 0 of a split chain is computed once, by its boundary item,
        // next to the summary pass (which then has no end-state items)
        e_in_c = use_tc && G >= 2;
        nA = G >= 2 ? chains * (G - 1 - (e_in_c ? 1 : 0)) : 0;
        nScan = G >= 2 ? chains : 0;
    } else {
        if (forced_s > 0) {
            forced_s &= 0xffff;
            if (forced_s < 1) return DN_ERR_INVALID_ARG;
            slots = d.H * ((n_c_max + d.N) / forced_s);
            if (slots > kMaxSlots) return DN_ERR_WORKSPACE;
        } else {
            slots = std::min<int64_t>(kAutoMaxSlots, d.H * (n_c_max + d.N));
        }
        nC = chains + slots;
        nA = slots;
        nScan = std::min<int64_t>(chains, slots);
    }
    // workspace layout
    const size_t off_items = 256;
    const size_t off_A = off_items + up256(nC * sizeof(Item) * (d.varlen ? 1 : 0));
    const size_t off_S = off_A + up256(nA * sizeof(Item) * (d.varlen ? 1 : 0));
    const size_t off_nc = off_S + up256(nScan * sizeof(Item) * (d.varlen ? 1 : 0));
    const size_t off_order = off_nc + up256(d.varlen ? d.N * 4 : 0);
    const size_t off_offs = off_order + up256(d.varlen ? d.N * 4 : 0);
    const size_t off_cum = off_offs + up256(d.varlen ? d.N * 16 : 0);
    const size_t off_P = off_cum + up256(d.varlen ? (d.N + 1) * 4 : 0);
    const size_t off_H = off_P + up256((size_t)slots * DK * DK * 4);
    const size_t off_SS = off_H + up256((size_t)slots * DK * DV * 4);
    // UT factors of every (chunk, head): chunks <= ceil(T / C) per row (+1 per sequence)
    const int64_t chunk_ub = d.varlen ? n_c_max + d.N : d.B * n_c_max;
    const size_t off_T = off_SS + up256((size_t)slots * DK * DV * 4);
    bytes = off_T + (use_tc ? (size_t)chunk_ub * d.H * (KDA ? kKdaUnitBytes : unit_bytes(GATED)) : 0);
    StreamWs ws;
    if ((st = get_ws(dev, stream, bytes, ws)) != DN_OK) return st;
    char* base = ws.buf;
    p.err = ws.flag;
    p.wsP = reinterpret_cast<float*>(base + off_P);
    p.wsH = reinterpret_cast<float*>(base + off_H);
    p.wsS = reinterpret_cast<float*>(base + off_SS);
    p.wsT = reinterpret_cast<uint8_t*>(base + off_T);
    Sched& sc = p.sched;
    std::memset(&sc, 0, sizeof sc);
    if (!d.varlen) {
        sc.list = 0;
        sc.B = (int)d.B;
        sc.T = (int)d.T;
        sc.H = (int)d.H;
        sc.n_chunks = (int)n_c_max;
        sc.G = G;
        sc.e_in_c = e_in_c ? 1 : 0;
        sc.s = s;
        sc.s0 = G >= 2 ? s0 : 0;
        g_last_G = G;
        g_last_s = s;
        g_last_s0 = G >= 2 && s0 > 0 ? s0 : s;
    } else {
        sc.list = 1;
        sc.B = 1;
        sc.T = (int)d.T;
        sc.H = (int)d.H;
        sc.itemsC = reinterpret_cast<const Item*>(base + off_items);
        sc.itemsA = reinterpret_cast<const Item*>(base + off_A);
        sc.itemsScan = reinterpret_cast<const Item*>(base + off_S);
        sc.counts = reinterpret_cast<const int*>(base);
        sc.cumchunks = reinterpret_cast<const int*>(base + off_cum);
        sc.cu = cu;
        sc.cu_mul = p.nh > 1 ? p.nh : 1;
        sc.N = (int)d.N;
        k_schedule<<<1, 1024, 0, stream>>>(
            cu, p.nh > 1 ? p.nh : 1, (int)d.N, (int)d.T, (int)d.H, forced_s, forced_s > 0 ? kMaxSlots : kAutoMaxSlots,
            sms, model, reinterpret_cast<Item*>(base + off_items),
            reinterpret_cast<Item*>(base + off_A), reinterpret_cast<Item*>(base + off_S),
            reinterpret_cast<int*>(base), reinterpret_cast<int*>(base + off_nc),
            reinterpret_cast<int*>(base + off_order), reinterpret_cast<int4*>(base + off_offs),
            reinterpret_cast<int*>(base + off_cum), ws.flag);
        g_last_G = -1;
        g_last_s = -1;
        g_last_s0 = -1;
    }
    CUtensorMap tp;
    if ((st = make_p_map(&tp, p.wsP, slots * DK, DK)) != DN_OK) return st;
    // one CTA per (chain, 8 state columns); 16 columns when that needs more than one wave
    auto launch_scan = [&]() {
        if (nScan * (DV / 8) <= sms)
            kS8<<<dim3((unsigned)nScan, DV / 8), scan_threads<DK, 8>(), smemS8, stream>>>(tp, p);
        else
            kS16<<<dim3((unsigned)nScan, DV / 16), scan_threads<DK, 16>(), smemS16, stream>>>(tp, p);
    };
    int launches = d.varlen ? 1 : 0;
    if (use_tc) {
        const int64_t units = chunk_ub * d.H;
        if (units > 0) {
            if constexpr (kKdaTc) {
                const int grid = (int)std::min<int64_t>(units, (int64_t)sms * 2);
                k_kda_prep<DK><<<grid, kThreads, smemPrep, stream>>>(p);
            } else {
                const int grid = (int)std::min<int64_t>(units, (int64_t)sms * prep_ctas_per_sm<GATED>());
                kPrep<<<grid, kPrepThreads, smemPrep, stream>>>(tq, tk, p);
            }
            ++launches;
        }
        if (e_in_c) {
            // run 0 of every chain (with outputs and its end state) on a second stream, next
            // to the summary pass, which leaves SMs free; the scan waits for both
            AuxStream aux;
            if ((st = get_aux(dev, stream, aux)) != DN_OK) return st;
            Params p0 = p;
            p0.sched.c_part = 1;
            if (cudaEventRecord(aux.fork, stream) != cudaSuccess ||
                cudaStreamWaitEvent(aux.stream, aux.fork, 0) != cudaSuccess)
                return DN_ERR_CUDA;
            kCt<<<(unsigned)chains, tc::kThreadsTc, smemCt, aux.stream>>>(tq, tk, tv, to, toc, p0);
            ++launches;
            if (cudaEventRecord(aux.join, aux.stream) != cudaSuccess) return DN_ERR_CUDA;
            if (nA > 0) { kAt<<<(unsigned)nA, tcs::kThreadsSum, smemAt, stream>>>(tk, tv, p); ++launches; }
            if (cudaStreamWaitEvent(stream, aux.join, 0) != cudaSuccess) return DN_ERR_CUDA;
            if (nScan > 0) { launch_scan(); ++launches; }
            Params p1 = p;
            p1.sched.c_part = 2;
            if (g_ev_start) cudaEventRecord(g_ev_start, stream);
            kCt<<<(unsigned)(chains * (G - 1)), tc::kThreadsTc, smemCt, stream>>>(tq, tk, tv, to, toc, p1);
            ++launches;
            if (g_ev_stop) cudaEventRecord(g_ev_stop, stream);
        } else {
            if (nA > 0) { kAt<<<(unsigned)nA, tcs::kThreadsSum, smemAt, stream>>>(tk, tv, p); ++launches; }
            if (nScan > 0) { launch_scan(); ++launches; }
            if (g_ev_start) cudaEventRecord(g_ev_start, stream);
            if (nC > 0) { kCt<<<(unsigned)nC, tc::kThreadsTc, smemCt, stream>>>(tq, tk, tv, to, toc, p); ++launches; }
            if (g_ev_stop) cudaEventRecord(g_ev_stop, stream);
        }
    } else {
        if (nA > 0) { kA<<<(unsigned)nA, kThreads, smemA, stream>>>(p); ++launches; }
        if (nScan > 0) { launch_scan(); ++launches; }
        if (g_ev_start) cudaEventRecord(g_ev_start, stream);
        if (nC > 0) { kC<<<(unsigned)nC, kThreads, smemC, stream>>>(p); ++launches; }
        if (g_ev_stop) cudaEventRecord(g_ev_stop, stream);
    }
    g_last_launches = launches;
    if (cudaGetLastError() != cudaSuccess) return DN_ERR_CUDA;
    return DN_OK;
}

// Kimi Delta Attention (a log decay per key channel): bf16 only; one load stage at d_k = 128
// (its per-channel gate tile takes the room of the second)
dn_status dispatch_kda(Params& p, const Dims& d, int dev, int sms, cudaStream_t stream, int forced_s,
                       const int* cup) {
    const int64_t dk = d.dk, dv = d.dv;
    if (dk == 128 && dv == 128)
        return launch<__nv_bfloat16, 128, 128, 1, false, true>(p, d, dev, sms, stream, forced_s, cup);
    if (dk == 128 && dv == 64)
        return launch<__nv_bfloat16, 128, 64, 1, false, true>(p, d, dev, sms, stream, forced_s, cup);
    if (dk == 64 && dv == 128)
        return launch<__nv_bfloat16, 64, 128, 2, false, true>(p, d, dev, sms, stream, forced_s, cup);
    return launch<__nv_bfloat16, 64, 64, 2, false, true>(p, d, dev, sms, stream, forced_s, cup);
}

template <bool GATED>
dn_status dispatch(Params& p, const Dims& d, int dev, int sms, cudaStream_t stream, int forced_s,
                   const int* cup, int32_t dt) {
    const int64_t dk = d.dk, dv = d.dv;
    if (dt == DN_F32) return launch<float, 64, 64, 1, GATED>(p, d, dev, sms, stream, forced_s, cup);
    if (dk == 128 && dv == 128)
        return launch<__nv_bfloat16, 128, 128, 2, GATED>(p, d, dev, sms, stream, forced_s, cup);
    if (dk == 128 && dv == 64)
        return launch<__nv_bfloat16, 128, 64, 2, GATED>(p, d, dev, sms, stream, forced_s, cup);
    if (dk == 64 && dv == 128)
        return launch<__nv_bfloat16, 64, 128, 2, GATED>(p, d, dev, sms, stream, forced_s, cup);
    return launch<__nv_bfloat16, 64, 64, 2, GATED>(p, d, dev, sms, stream, forced_s, cup);
}

// gate: Gated DeltaNet's log decay [B, T, H] fp32, or null for DeltaNet; with kda, Kimi
// Delta Attention's log decay per key channel [B, T, H, d_k] fp32.
// nh: delta-rule writes per token (Gated Delta Product; 1 otherwise): k, v and beta hold
// T * nh rows, q, gate and out T rows, cu_seqlens counts tokens.
// cs: chunk-start states [rows, H, d_k, d_v] fp32, or null.
dn_status fwd_impl(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                   const dn_tensor* beta, const dn_tensor* gate, const dn_tensor* s0,
                   const dn_tensor* cu, int chunk, dn_tensor* out, dn_tensor* sT,
                   void* stream_ptr, int forced_s, int nh = 1, dn_tensor* cs = nullptr,
                   bool kda = false) {
    if (!q || !k || !v || !beta || !out) return DN_ERR_INVALID_ARG;
    if (q->ndim != 4 || k->ndim != 4 || v->ndim != 4 || out->ndim != 4) return DN_ERR_INVALID_ARG;
    if (forced_s < 0 || nh < 1 || (nh > 1 && !gate)) return DN_ERR_INVALID_ARG;
    const int64_t B = q->shape[0], T = q->shape[1], H = q->shape[2], dk = q->shape[3];
    const int64_t dv = v->shape[3];
    if (B < 0 || T < 0 || H < 1 || dk < 1 || dv < 1) return DN_ERR_INVALID_ARG;
    if (nh > 1024 || T * nh >= (int64_t(1) << 31)) return DN_ERR_INVALID_ARG;
    const int64_t Tw = T * nh;  // rows of k, v, beta
    const int64_t kd[4] = {B, Tw, H, dk}, vd[4] = {B, Tw, H, dv}, bd[3] = {B, Tw, H};
    const int64_t od[4] = {B, T, H, dv}, gd[3] = {B, T, H};
    if (!shape_eq(k, 4, kd) || !shape_eq(v, 4, vd) || !shape_eq(out, 4, od) ||
        !shape_eq(beta, 3, bd))
        return DN_ERR_INVALID_ARG;
    const int32_t dt = q->dtype;
    if ((dt != DN_BF16 && dt != DN_F32) || k->dtype != dt || v->dtype != dt || out->dtype != dt)
        return DN_ERR_INVALID_ARG;
    if (beta->dtype != DN_F32) return DN_ERR_INVALID_ARG;
    if (!token_tensor_ok(q) || !token_tensor_ok(k) || !token_tensor_ok(v) || !token_tensor_ok(out))
        return DN_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
        if (beta->stride[i] < 0) return DN_ERR_INVALID_ARG;
    if (numel(beta) > 0 && (!beta->data || (reinterpret_cast<uintptr_t>(beta->data) & 3)))
        return DN_ERR_INVALID_ARG;
    if (kda) {
        // one log decay per key channel, rows of d_k fp32 read in 16-byte pieces
        const int64_t gk[4] = {B, T, H, dk};
        if (!gate || nh != 1 || !shape_eq(gate, 4, gk) || gate->dtype != DN_F32) return DN_ERR_INVALID_ARG;
        if (!token_tensor_ok(gate)) return DN_ERR_INVALID_ARG;
        if (dt != DN_BF16) return DN_ERR_UNSUPPORTED;
    } else if (gate) {
        if (!shape_eq(gate, 3, gd) || gate->dtype != DN_F32) return DN_ERR_INVALID_ARG;
        for (int i = 0; i < 3; ++i)
            if (gate->stride[i] < 0) return DN_ERR_INVALID_ARG;
        if (numel(gate) > 0 && (!gate->data || (reinterpret_cast<uintptr_t>(gate->data) & 3)))
            return DN_ERR_INVALID_ARG;
    }
    if (B * Tw >= (int64_t(1) << 31) || H >= 65536) return DN_ERR_INVALID_ARG;

    int64_t N = B;
    const bool varlen = cu != nullptr;
    if (varlen) {
        if (cu->ndim != 1 || cu->dtype != DN_I32 || cu->shape[0] < 1 || cu->stride[0] != 1 ||
            !cu->data || (reinterpret_cast<uintptr_t>(cu->data) & 3))
            return DN_ERR_INVALID_ARG;
        if (B != 1) return DN_ERR_INVALID_ARG;
        N = cu->shape[0] - 1;
        if (N >= (int64_t(1) << 24)) return DN_ERR_INVALID_ARG;
    }
    const int64_t sd[4] = {N, H, dk, dv};
    if (s0 && (!shape_eq(s0, 4, sd) || !state_tensor_ok(s0, dv))) return DN_ERR_INVALID_ARG;
    if (sT && (!shape_eq(sT, 4, sd) || !state_tensor_ok(sT, dv))) return DN_ERR_INVALID_ARG;
    if (cs) {
        // one row per chunk: exactly B * ceil(T / C) for a dense batch; for packed input at
        // least ceil(T / C) + N, which bounds the sum of ceil(L_n / C) over the sequences
        const int64_t n_c = (Tw + kChunk - 1) / kChunk;
        const int64_t need = varlen ? n_c + N : B * n_c;
        if (cs->ndim != 4 || cs->shape[1] != H || cs->shape[2] != dk || cs->shape[3] != dv ||
            !state_tensor_ok(cs, dv))
            return DN_ERR_INVALID_ARG;
        if (varlen ? cs->shape[0] < need : cs->shape[0] != need) return DN_ERR_INVALID_ARG;
    }

    if (chunk != kChunk) return DN_ERR_UNSUPPORTED;
    const bool bf16_ok = (dk == 64 || dk == 128) && (dv == 64 || dv == 128);
    const bool f32_ok = dk == 64 && dv == 64;
    if (dt == DN_BF16 ? !bf16_ok : !f32_ok) return DN_ERR_UNSUPPORTED;

    // aliasing: outputs against inputs and each other
    const dn_tensor* ins[7] = {q, k, v, beta, gate, s0, cu};
    for (const dn_tensor* o : {static_cast<const dn_tensor*>(out), static_cast<const dn_tensor*>(sT)}) {
        if (!o) continue;
        for (const dn_tensor* in : ins)
            if (in && overlap(o, in)) return DN_ERR_ALIAS;
    }
    if (sT && overlap(out, sT)) return DN_ERR_ALIAS;
    if (cs) {
        for (const dn_tensor* in : ins)
            if (in && overlap(cs, in)) return DN_ERR_ALIAS;
        if (overlap(cs, out) || (sT && overlap(cs, sT))) return DN_ERR_ALIAS;
    }

    int dev = 0, sms = 0;
    dn_status st = device_check(dev, sms);
    if (st != DN_OK) return st;
    if (N == 0) return DN_OK;

    Params p;
    std::memset(&p, 0, sizeof p);
    p.wait_ns = g_wait_ns;
    p.stall_chunk = g_stall_chunk;
    p.q = q->data; p.k = k->data; p.v = v->data; p.o = out->data;
    p.beta = static_cast<const float*>(beta->data);
    p.s0 = s0 && numel(s0) ? static_cast<const float*>(s0->data) : nullptr;
    p.sT = sT && numel(sT) ? static_cast<float*>(sT->data) : nullptr;
    p.q_sb = q->stride[0]; p.q_st = q->stride[1]; p.q_sh = q->stride[2];
    p.k_sb = k->stride[0]; p.k_st = k->stride[1]; p.k_sh = k->stride[2];
    p.v_sb = v->stride[0]; p.v_st = v->stride[1]; p.v_sh = v->stride[2];
    p.o_sb = out->stride[0]; p.o_st = out->stride[1]; p.o_sh = out->stride[2];
    p.b_sb = beta->stride[0]; p.b_st = beta->stride[1]; p.b_sh = beta->stride[2];
    if (gate) {
        p.g = static_cast<const float*>(gate->data);
        p.g_sb = gate->stride[0]; p.g_st = gate->stride[1]; p.g_sh = gate->stride[2];
    }
    if (s0) { p.s0_sn = s0->stride[0]; p.s0_sh = s0->stride[1]; }
    if (sT) { p.sT_sn = sT->stride[0]; p.sT_sh = sT->stride[1]; }

    p.nh = nh;
    if (cs && numel(cs)) {
        p.cs = static_cast<float*>(cs->data);
        p.cs_sc = cs->stride[0];
        p.cs_sh = cs->stride[1];
        p.cs_rows = cs->shape[0];
    }
    Dims d{B, Tw, H, dk, dv, N, varlen};  // items count k/v/beta rows
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    const int* cup = varlen ? static_cast<const int*>(cu->data) : nullptr;
    if (kda) return dispatch_kda(p, d, dev, sms, stream, forced_s, cup);
    if (gate) return dispatch<true>(p, d, dev, sms, stream, forced_s, cup, dt);
    return dispatch<false>(p, d, dev, sms, stream, forced_s, cup, dt);
}

}  // namespace

extern "C" {

dn_status deltanet_fwd(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                       const dn_tensor* beta, const dn_tensor* initial_state,
                       const dn_tensor* cu_seqlens, int chunk_size, dn_tensor* out,
                       dn_tensor* final_state, void* stream) {
    return fwd_impl(q, k, v, beta, nullptr, initial_state, cu_seqlens, chunk_size, out,
                    final_state, stream, 0);
}

dn_status deltanet_fwd_ex(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                          const dn_tensor* beta, const dn_tensor* initial_state,
                          const dn_tensor* cu_seqlens, int chunk_size, dn_tensor* out,
                          dn_tensor* final_state, void* stream, int seg_chunks) {
    return fwd_impl(q, k, v, beta, nullptr, initial_state, cu_seqlens, chunk_size, out,
                    final_state, stream, seg_chunks);
}

dn_status gated_deltanet_fwd(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                             const dn_tensor* beta, const dn_tensor* g,
                             const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                             int chunk_size, dn_tensor* out, dn_tensor* final_state,
                             void* stream) {
    if (!g) return DN_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, beta, g, initial_state, cu_seqlens, chunk_size, out, final_state,
                    stream, 0);
}

dn_status gated_deltanet_fwd_ex(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                                const dn_tensor* beta, const dn_tensor* g,
                                const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                                int chunk_size, dn_tensor* out, dn_tensor* final_state,
                                void* stream, int seg_chunks) {
    if (!g) return DN_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, beta, g, initial_state, cu_seqlens, chunk_size, out, final_state,
                    stream, seg_chunks);
}

dn_status deltanet_fwd_states(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                              const dn_tensor* beta, const dn_tensor* g,
                              const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                              int chunk_size, dn_tensor* out, dn_tensor* final_state,
                              dn_tensor* chunk_states, void* stream, int seg_chunks) {
    if (!chunk_states) return DN_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, beta, g, initial_state, cu_seqlens, chunk_size, out, final_state,
                    stream, seg_chunks, 1, chunk_states);
}

dn_status gated_deltaproduct_fwd(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                                 const dn_tensor* beta, const dn_tensor* g,
                                 const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                                 int n_h, int chunk_size, dn_tensor* out,
                                 dn_tensor* final_state, void* stream) {
    if (!g) return DN_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, beta, g, initial_state, cu_seqlens, chunk_size, out, final_state,
                    stream, 0, n_h);
}

dn_status gated_deltaproduct_fwd_ex(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v,
                                    const dn_tensor* beta, const dn_tensor* g,
                                    const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                                    int n_h, int chunk_size, dn_tensor* out,
                                    dn_tensor* final_state, void* stream, int seg_chunks) {
    if (!g) return DN_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, beta, g, initial_state, cu_seqlens, chunk_size, out, final_state,
                    stream, seg_chunks, n_h);
}

dn_status kda_fwd(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v, const dn_tensor* beta,
                  const dn_tensor* g, const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                  int chunk_size, dn_tensor* out, dn_tensor* final_state, void* stream) {
    if (!g) return DN_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, beta, g, initial_state, cu_seqlens, chunk_size, out, final_state,
                    stream, 0, 1, nullptr, true);
}

dn_status kda_fwd_ex(const dn_tensor* q, const dn_tensor* k, const dn_tensor* v, const dn_tensor* beta,
                     const dn_tensor* g, const dn_tensor* initial_state, const dn_tensor* cu_seqlens,
                     int chunk_size, dn_tensor* out, dn_tensor* final_state, void* stream,
                     int seg_chunks) {
    if (!g) return DN_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, beta, g, initial_state, cu_seqlens, chunk_size, out, final_state,
                    stream, seg_chunks, 1, nullptr, true);
}

const char* deltanet_status_string(dn_status s) {
    switch (s) {
        case DN_OK: return "DN_OK";
        case DN_ERR_INVALID_ARG: return "DN_ERR_INVALID_ARG: bad shape, dtype, stride, alignment or pointer";
        case DN_ERR_UNSUPPORTED: return "DN_ERR_UNSUPPORTED: chunk size, head dims or device not supported";
        case DN_ERR_ALIAS: return "DN_ERR_ALIAS: an output overlaps an input or another output";
        case DN_ERR_CUDA: return "DN_ERR_CUDA: CUDA runtime or launch error";
        case DN_ERR_WORKSPACE: return "DN_ERR_WORKSPACE: workspace allocation failed or limit exceeded";
        case DN_ERR_SEQLENS: return "DN_ERR_SEQLENS: invalid cu_seqlens contents";
        case DN_ERR_TIMEOUT: return "DN_ERR_TIMEOUT: a bounded device wait gave up";
    }
    return "unknown dn_status";
}

dn_status deltanet_get_error(void* stream_ptr) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DN_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return DN_ERR_CUDA;
    // the no-alloc entry point's error word (one per device), then this stream's flag
    int h = 0;
    if (dn_noalloc_take_error(dev, &h) != 0) return DN_ERR_CUDA;
    int* flag = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_ws.find(std::make_pair(dev, stream));
        if (it != g_ws.end()) flag = it->second.flag;
    }
    if (flag) {
        int f = 0;
        if (cudaMemcpy(&f, flag, sizeof f, cudaMemcpyDeviceToHost) != cudaSuccess) return DN_ERR_CUDA;
        if (f != 0 && cudaMemset(flag, 0, sizeof f) != cudaSuccess) return DN_ERR_CUDA;
        if (h == 0) h = f;
    }
    if (h == kErrSeqlens) return DN_ERR_SEQLENS;
    if (h == kErrTimeout) return DN_ERR_TIMEOUT;
    return DN_OK;
}

void deltanet_test_set_wait(unsigned long long wait_ns, int stall_chunk) {
    g_wait_ns = wait_ns;
    g_stall_chunk = stall_chunk > 0 ? stall_chunk : 0;
}

}  // extern "C"

void dn_wait_settings(unsigned long long* wait_ns, int* stall_chunk) {
    *wait_ns = g_wait_ns;
    *stall_chunk = g_stall_chunk;
}

extern "C" {

void deltanet_release_workspace(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    int cur = 0;
    cudaGetDevice(&cur);
    for (auto& kv : g_ws) {
        cudaSetDevice(kv.first.first);
        cudaDeviceSynchronize();
        if (kv.second.buf) cudaFree(kv.second.buf);
        if (kv.second.flag) cudaFree(kv.second.flag);
    }
    g_ws.clear();
    cudaSetDevice(cur);
}

#ifdef DN_TRACE
int dn_trace_copy(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, tc::g_dn_trace, sizeof(tc::g_dn_trace)) == cudaSuccess ? 0 : 1;
}
int dn_trace_copy_prep(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, g_dn_trace_prep, sizeof(g_dn_trace_prep)) == cudaSuccess ? 0 : 1;
}
int dn_trace_copy_sum(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, tcs::g_dn_trace_sum, sizeof(tcs::g_dn_trace_sum)) == cudaSuccess ? 0 : 1;
}
int dn_trace_copy_kda(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, g_dn_trace_kda, sizeof(g_dn_trace_kda)) == cudaSuccess ? 0 : 1;
}
int dn_trace_copy_scan(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, g_dn_trace_scan, sizeof(g_dn_trace_scan)) == cudaSuccess ? 0 : 1;
}
#endif

void deltanet_last_schedule(int* segments_per_chain, int* chunks_per_segment, int* chunks_first_segment) {
    if (chunks_first_segment) *chunks_first_segment = g_last_s0;
    if (segments_per_chain) *segments_per_chain = g_last_G;
    if (chunks_per_segment) *chunks_per_segment = g_last_s;
}

int deltanet_last_launches(void) { return g_last_launches; }

void deltanet_set_kernel_events(void* start_event, void* stop_event) {
    g_ev_start = static_cast<cudaEvent_t>(start_event);
    g_ev_stop = static_cast<cudaEvent_t>(stop_event);
}

}  // extern "C"
