// Tensor-core (tcgen05 / TMEM / TMA) chain kernel for bf16, d_k = d_v = 128.
//
// Same per-chunk algorithm as dn_chain.cuh ("Linear Attention, Visualized",
// DeltaNet, "Complete per-chunk algorithm"), evaluated in the transposed
// domain so that every tensor-core product has M = 128:
//   G   = [Q; K] K^T                      (rows: 64 queries, then 64 keys)
//   P   = (Q K^T) o M_c from the query rows of G (output runs only)
//   T   = (I + B L)^{-1} B               (from the UT pre-pass, dn_prep.cuh)
//   W^T = K^T T^T,  U^T = V^T T^T
//   Z^T = U^T - S^T W^T                  (accumulated into U^T's columns)
//   O^T = S^T Q^T + Z^T P^T
//   S^T <- S^T + Z^T K
// S^T (d_v lanes x d_k columns, fp32) lives in tensor memory for the whole run;
// a bf16 copy in shared memory feeds the next chunk's products.
//
// Warp roles (512 threads):
//   warps 0-7   chain epilogue: Z^T -> bf16, S^T -> bf16, O -> global
//   warps 8-11  chunk-parallel epilogue: W^T -> bf16 rows; G -> P
//   warp 12     issues the state-chain products (Z, O, S updates), one thread;
//               owns the tensor-memory allocation
//   warp 13     TMA loads of q, k (3-stage ring), one thread
//   warp 14     issues the chunk-parallel products (G, W^T, U^T), one thread
//   warp 15     TMA loads of v and bulk copies of T (2-stage ring), one thread
// The two issuers run independently, so the chunk-parallel work of chunk
// r+1 overlaps the state chain of chunk r.  Buffers that outlive one chunk
// are double-buffered with one "free" barrier per buffer.  Every wait on an
// mbarrier is bounded; on time-out the CTA drains, frees its tensor memory
// and reports DN_ERR_TIMEOUT through the error flag.
#pragma once

#include "dn_common.cuh"
#include "dn_sm100.cuh"

namespace dn {
namespace tc {

using namespace sm100;

constexpr int D = 128;
constexpr int kThreadsTc = 512;
constexpr int kChainMmaWarp = 12;
constexpr int kTmaWarp = 13;
constexpr int kParMmaWarp = 14;
constexpr int kTmaBWarp = 15;

// shared memory (byte offsets from a 1024-aligned base)
//   ring A (q, k): 3 stages of [Q d0-63 | K d0-63 | Q d64-127 | K d64-127]
//   ring B (v, T): 2 stages of [V d0-63 | V d64-127 | T]
constexpr int NA = 3, NB = 2;
constexpr int A_STAGE = 32768;
constexpr int OFF_B = NA * A_STAGE;
constexpr int B_STAGE = 24576, B_T = 16384;
constexpr int OFF_WB = OFF_B + NB * B_STAGE;   // W^T rows (d_k rows of 64 tokens)
constexpr int OFF_PB = OFF_WB + 16384;         // P rows
constexpr int OFF_ZB = OFF_PB + 8192;          // Z^T rows
constexpr int OFF_SBF = OFF_ZB + 16384;        // S^T rows, bf16
constexpr int OFF_BAR = OFF_SBF + 32768;
constexpr int NBAR = 26;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM_USED = OFF_MISC + 64;
constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// tensor-memory columns (512 allocated): S^T, O^T, 2 x U^T/Z^T, 2 x W^T, G
constexpr uint32_t TM_S = 0, TM_O = 128, TM_ZU = 192, TM_WT = 320, TM_G = 448;

// Barriers of a ring or of a double buffer come one per slot; a waiter on slot
// s for chunk r waits for that slot's (r / slots)-th completion.
enum : int {
    B_FULLA = 0,     // +3: q, k of a stage landed
    B_EMPTYA = 3,    // +3: stage of ring A consumed by both issuers
    B_FULLB = 6,     // +2: v, T landed
    B_EMPTYB = 8,    // +2: stage of ring B consumed
    B_GFULL = 10,    // G ready in TMEM
    B_GFREE = 11,    // G read out (P written)
    B_WUFULL = 12,   // +2: W^T, U^T ready in TMEM
    B_WFULL = 14,    // W^T rows written to shared memory
    B_C1A = 15,      // Z^T = U^T - S^T W^T complete
    B_ZFULL = 16,    // Z^T (bf16) written
    B_SFULL = 17,    // S^T updated
    B_OFULL = 18,    // O^T complete (P consumed)
    B_SBF = 19,      // bf16 copy of S^T written
    B_OFREE = 20,    // O^T read out
    B_ZFREE = 21,    // +2: U^T / Z^T columns read out
    B_WTFREE = 23,   // +2: W^T columns read out
};

// Optional timeline of CTA 0 (build with -DDN_TRACE): globaltimer stamps per
// chunk and pipeline event, read back with dn_trace_copy().
#ifdef DN_TRACE
static __device__ unsigned long long g_dn_trace[64 * 32];
#define DN_TR(cond, r, slot)                                                          \
    do {                                                                              \
        if ((cond) && blockIdx.x == 0 && (r) < 64 && (threadIdx.x & 31) == 0)          \
            g_dn_trace[(r) * 32 + (slot)] = globaltimer();                            \
    } while (0)
#else
#define DN_TR(cond, r, slot) \
    do {                     \
    } while (0)
#endif

// N fp32 values (N = 32 or 64) -> swizzled 16-byte chunks (bf16) of row r from column c0.
template <int N>
__device__ __forceinline__ void st_row_bf16(uint8_t* tile, int r, int c0, const uint32_t* v) {
#pragma unroll
    for (int k = 0; k < N / 8; ++k) {
        uint4 u;
        u.x = pack_bf16(__uint_as_float(v[8 * k + 0]), __uint_as_float(v[8 * k + 1]));
        u.y = pack_bf16(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3]));
        u.z = pack_bf16(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5]));
        u.w = pack_bf16(__uint_as_float(v[8 * k + 6]), __uint_as_float(v[8 * k + 7]));
        *reinterpret_cast<uint4*>(tile + swz128(r, c0 + 8 * k)) = u;
    }
}

template <bool HAS_Q>
__global__ void __launch_bounds__(kThreadsTc, 1)
    k_tc_chain(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int n_items = HAS_Q ? count_C(p.sched) : count_A(p.sched);
    if ((int)blockIdx.x >= n_items) return;
    int mode = kModeOut;
    const Item it = HAS_Q ? item_C(p.sched, blockIdx.x) : item_A(p.sched, blockIdx.x, mode);
    const bool has_v = mode != kModeP;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 8);
    uint8_t* Wb = smem + OFF_WB;
    uint8_t* Zb = smem + OFF_ZB;
    uint8_t* Sbf = smem + OFF_SBF;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NA; ++s) {
            mbar_init(&bars[B_FULLA + s], 1);
            mbar_init(&bars[B_EMPTYA + s], 2);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[B_FULLB + s], 1);
            mbar_init(&bars[B_EMPTYB + s], 1);
            mbar_init(&bars[B_WUFULL + s], 1);
            mbar_init(&bars[B_ZFREE + s], 256);
            mbar_init(&bars[B_WTFREE + s], 128);
        }
        mbar_init(&bars[B_GFULL], 1);
        mbar_init(&bars[B_GFREE], 64);
        mbar_init(&bars[B_WFULL], 128);
        mbar_init(&bars[B_C1A], 1);
        mbar_init(&bars[B_ZFULL], 256);
        mbar_init(&bars[B_SFULL], 1);
        mbar_init(&bars[B_OFULL], 1);
        mbar_init(&bars[B_SBF], 256);
        mbar_init(&bars[B_OFREE], 256);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kChainMmaWarp) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int ntok = it.tok1 - it.tok0;
    const int nch = (ntok + kChunk - 1) / kChunk;

    // start state and destination of the run
    const float* x_in = nullptr;
    float* x_out = nullptr;
    bool identity = false;
    const float* s0 = p.s0 ? p.s0 + it.seq * p.s0_sn + it.head * p.s0_sh : nullptr;
    if (mode == kModeOut) {
        x_in = it.g == 0 ? s0 : p.wsS + (int64_t)(it.slot + it.g - 1) * D * D;
        if (it.g == it.G - 1 && p.sT) x_out = p.sT + it.seq * p.sT_sn + it.head * p.sT_sh;
    } else if (mode == kModeEnd) {
        x_in = s0;
        x_out = p.wsH + (int64_t)it.slot * D * D;
    } else if (mode == kModeH) {
        x_out = p.wsH + (int64_t)(it.slot + it.g) * D * D;
    } else {
        identity = true;
        x_out = p.wsP + (int64_t)(it.slot + it.g) * D * D;
    }

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ ring A: q, k
        if (lane == 0 && nch > 0) {
            const uint32_t bytes = (HAS_Q ? 16384u : 0u) + 16384u;
            int issued = 0;
            for (int r = 0; r < nch; ++r) {
                const int s = r % NA;
                if (r >= NA && !mbar_wait(&bars[B_EMPTYA + s], ((r / NA) - 1) & 1, abort_flag)) break;
                mbar_expect_tx(&bars[B_FULLA + s], bytes);
                uint8_t* st = smem + s * A_STAGE;
                const int t0 = it.tok0 + r * kChunk;
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    if (HAS_Q) tma_load_4d(st + a * 16384, &tq, &bars[B_FULLA + s], a * 64, it.head, t0, it.b);
                    tma_load_4d(st + a * 16384 + 8192, &tk, &bars[B_FULLA + s], a * 64, it.head, t0, it.b);
                }
                issued = r + 1;
                DN_TR(true, r, 24);
            }
            // the last loads issued must have landed before the CTA may exit
            for (int r = issued - NA < 0 ? 0 : issued - NA; r < issued; ++r)
                mbar_wait(&bars[B_FULLA + (r % NA)], (r / NA) & 1, abort_flag, 200000000ull);
        }
    } else if (warp == kTmaBWarp) {
        // ------------------------------------------------------------ ring B: v, T
        if (lane == 0 && nch > 0) {
            const uint32_t bytes = (has_v ? 16384u : 0u) + 8192u;
            int issued = 0;
            for (int r = 0; r < nch; ++r) {
                const int s = r & 1;
                if (r >= 2 && !mbar_wait(&bars[B_EMPTYB + s], ((r >> 1) - 1) & 1, abort_flag)) break;
                mbar_expect_tx(&bars[B_FULLB + s], bytes);
                uint8_t* st = smem + OFF_B + s * B_STAGE;
                const int t0 = it.tok0 + r * kChunk;
                if (has_v) {
#pragma unroll
                    for (int a = 0; a < 2; ++a)
                        tma_load_4d(st + a * 8192, &tv, &bars[B_FULLB + s], a * 64, it.head, t0, it.b);
                }
                bulk_load(st + B_T, p.wsT + ((size_t)(it.cbase + r) * p.sched.H + it.head) * 8192, 8192,
                          &bars[B_FULLB + s]);
                issued = r + 1;
            }
            for (int r = issued - 2 < 0 ? 0 : issued - 2; r < issued; ++r)
                mbar_wait(&bars[B_FULLB + (r & 1)], (r >> 1) & 1, abort_flag, 200000000ull);
        }
    } else if (warp == kParMmaWarp) {
        // ------------------------------------------------------------ chunk-parallel products
        if (lane == 0 && nch > 0) {
            const uint32_t sb = saddr(smem);
            const uint32_t i_g = idesc_bf16(128, 64, false, false);
            const uint32_t i_tt = idesc_bf16(128, 64, true, false);
            // descriptors at offset 0; per-step offsets are added in 16-byte units
            const uint64_t dQK = sdesc(sb, 16, 1024);                  // K-major [Q;K] / K rows
            const uint64_t dKT = sdesc(sb + 8192, 16384, 1024);        // K^T, MN-major
            const uint64_t dVT = sdesc(sb + OFF_B, 8192, 1024);        // V^T, MN-major
            const uint64_t dT = sdesc(sb + OFF_B + B_T, 16, 1024);     // T^T, K-major
            for (int r = 0; r < nch; ++r) {
                const int sa = r % NA, s = r & 1;
                const uint64_t sta = (uint64_t)((sa * A_STAGE) >> 4);
                const uint64_t stb = (uint64_t)((s * B_STAGE) >> 4);
                if (!mbar_wait(&bars[B_FULLA + sa], (r / NA) & 1, abort_flag)) break;
                if (HAS_Q) {
                    // G = [Q; K] K^T (only the query rows are used: P)
                    if (r >= 1 && !mbar_wait(&bars[B_GFREE], (r - 1) & 1, abort_flag)) break;
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint64_t o = sta + (uint64_t)(((j >> 2) * 16384 + (j & 3) * 32) >> 4);
                        umma_bf16(tmem + TM_G, dQK + o, dQK + o + (8192 >> 4), i_g, j > 0);
                    }
                    umma_commit(&bars[B_GFULL]);
                }
                // W^T = K^T T^T, U^T = V^T T^T once this parity's W^T and U^T columns are free
                if (!mbar_wait(&bars[B_FULLB + s], (r >> 1) & 1, abort_flag)) break;
                if (r >= 2 && (!mbar_wait(&bars[B_WTFREE + s], ((r >> 1) - 1) & 1, abort_flag) ||
                               !mbar_wait(&bars[B_ZFREE + s], ((r >> 1) - 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    umma_bf16(tmem + TM_WT + s * 64, dKT + sta + (uint64_t)((j * 2048) >> 4),
                              dT + stb + (uint64_t)((j * 32) >> 4), i_tt, j > 0);
                if (has_v) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_bf16(tmem + TM_ZU + s * 64, dVT + stb + (uint64_t)((j * 2048) >> 4),
                                  dT + stb + (uint64_t)((j * 32) >> 4), i_tt, j > 0);
                }
                umma_commit(&bars[B_WUFULL + s]);
                umma_commit(&bars[B_EMPTYB + s]);
                umma_commit(&bars[B_EMPTYA + sa]);
                DN_TR(true, r, 5);
            }
        }
    } else if (warp == kChainMmaWarp) {
        // ------------------------------------------------------------ state-chain products
        if (lane == 0 && nch > 0) {
            const uint32_t sb = saddr(smem);
            const uint32_t i_c1a = idesc_bf16(128, 64, false, true, true);
            const uint32_t i_c1b = idesc_bf16(128, 64, false, false);
            const uint32_t i_c3 = idesc_bf16(128, 128, false, true);
            const uint32_t i_c2 = idesc_bf16(128, 64, false, false);
            const uint64_t dS = sdesc(sb + OFF_SBF, 16, 1024);   // S^T, K-major
            const uint64_t dW = sdesc(sb + OFF_WB, 8192, 1024);  // W^T rows, MN-major (64 tokens)
            const uint64_t dQ = sdesc(sb, 16, 1024);             // Q^T, K-major
            const uint64_t dZ = sdesc(sb + OFF_ZB, 16, 1024);    // Z^T, K-major
            const uint64_t dK = sdesc(sb + 8192, 16384, 1024);   // K, MN-major
            const uint64_t dP = sdesc(sb + OFF_PB, 16, 1024);    // P^T, K-major
            for (int r = 0; r < nch; ++r) {
                const int sa = r % NA, s = r & 1;
                const uint64_t sta = (uint64_t)((sa * A_STAGE) >> 4);
                DN_TR(true, r, 0);
                if (!mbar_wait(&bars[B_WFULL], r & 1, abort_flag) ||
                    !mbar_wait(&bars[B_SBF], r & 1, abort_flag)) break;
                tc_fence_after();
                // Z^T = U^T - S^T W^T
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint64_t o = (uint64_t)(((j >> 2) * 16384 + (j & 3) * 32) >> 4);
                    const uint64_t wo = (uint64_t)((j * 2048) >> 4);
                    umma_bf16(tmem + TM_ZU + s * 64, dS + o, dW + wo, i_c1a,
                              has_v ? 1u : (j > 0 ? 1u : 0u));
                }
                umma_commit(&bars[B_C1A]);
                DN_TR(true, r, 1);
                if (HAS_Q) {
                    if (!mbar_wait(&bars[B_OFREE], r & 1, abort_flag)) break;
                    tc_fence_after();
                    // O^T = S^T Q^T
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint64_t o = (uint64_t)(((j >> 2) * 16384 + (j & 3) * 32) >> 4);
                        umma_bf16(tmem + TM_O, dS + o, dQ + sta + o, i_c1b, j > 0);
                    }
                }
                DN_TR(true, r, 2);
                if (!mbar_wait(&bars[B_ZFULL], r & 1, abort_flag)) break;
                tc_fence_after();
                // S^T += Z^T K
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    umma_bf16(tmem + TM_S, dZ + (uint64_t)((j * 32) >> 4),
                              dK + sta + (uint64_t)((j * 2048) >> 4), i_c3, 1u);
                umma_commit(&bars[B_SFULL]);
                if (HAS_Q) {
                    // O^T += Z^T P^T
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_bf16(tmem + TM_O, dZ + (uint64_t)((j * 32) >> 4),
                                  dP + (uint64_t)((j * 32) >> 4), i_c2, 1u);
                    umma_commit(&bars[B_OFULL]);
                }
                umma_commit(&bars[B_EMPTYA + sa]);
                DN_TR(true, r, 4);
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ chunk-parallel epilogue
        const int q = warp - 8;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        for (int r = 0; r < nch; ++r) {
            const int s = r & 1;
            // W^T (TMEM, d_k lanes) -> bf16 rows of 64 tokens (an MN-major operand),
            // once the previous W^T rows are consumed
            if (r >= 1 && !__all_sync(0xffffffffu, mbar_wait(&bars[B_C1A], (r - 1) & 1, abort_flag))) break;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_WUFULL + s], (r >> 1) & 1, abort_flag))) break;
            DN_TR(q == 0, r, 13);
            tc_fence_after();
            {
                uint32_t v[64];
                tmem_ld64(tmem + lane_base + TM_WT + s * 64, v);
                tc_fence_before();
                mbar_arrive(&bars[B_WTFREE + s]);
                st_row_bf16<64>(Wb, 32 * q + lane, 0, v);
            }
            fence_async_smem();
            mbar_arrive(&bars[B_WFULL]);
            DN_TR(q == 0, r, 14);
            if (HAS_Q && q < 2) {
                // query rows of G: P = (Q K^T) o M_c (inclusive), bf16 rows i, once the
                // previous P is consumed
                if (r >= 1 && !__all_sync(0xffffffffu, mbar_wait(&bars[B_OFULL], (r - 1) & 1, abort_flag))) break;
                if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_GFULL], r & 1, abort_flag))) break;
                DN_TR(q == 0, r, 8);
                tc_fence_after();
                const int i = 32 * q + lane;
                uint32_t v[64];
                tmem_ld64(tmem + lane_base + TM_G, v);
                tc_fence_before();
                mbar_arrive(&bars[B_GFREE]);
#pragma unroll
                for (int jj = 0; jj < 64; ++jj)
                    if (jj > i) v[jj] = 0u;
                st_row_bf16<64>(smem + OFF_PB, i, 0, v);
                fence_async_smem();
                DN_TR(q == 0, r, 9);
            }
        }
    } else {
        // ------------------------------------------------------------ chain epilogue
        const int wq = warp & 3, h = warp >> 2;
        const int d = 32 * wq + lane;  // d_v row of S^T, Z^T, O^T
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        {
            uint32_t v[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const int a = 64 * h + c;
                float x = 0.f;
                if (x_in) x = x_in[(int64_t)a * D + d];
                else if (identity) x = (a == d) ? 1.f : 0.f;
                v[c] = __float_as_uint(x);
            }
            if (nch == 0) {
                if (x_out)
                    for (int c = 0; c < 64; ++c) x_out[(int64_t)(64 * h + c) * D + d] = __uint_as_float(v[c]);
            } else {
                tmem_st32(tmem + lane_base + TM_S + 64 * h, *reinterpret_cast<uint32_t(*)[32]>(v));
                tmem_st32(tmem + lane_base + TM_S + 64 * h + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                st_row_bf16<64>(Sbf + h * 16384, d, 0, v);
            }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&bars[B_SBF]);
        if (HAS_Q) mbar_arrive(&bars[B_OFREE]);
        __nv_bfloat16* og = static_cast<__nv_bfloat16*>(p.o) + it.b * p.o_sb + it.head * p.o_sh;
        for (int r = 0; r < nch; ++r) {
            const int s = r & 1;
            // Z^T -> bf16 operand
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_C1A], r & 1, abort_flag))) break;
            DN_TR(warp == 0, r, 16);
            tc_fence_after();
            {
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + TM_ZU + s * 64 + 32 * h, v);
                st_row_bf16<32>(Zb, d, 32 * h, v);
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_ZFULL]);
            mbar_arrive(&bars[B_ZFREE + s]);
            DN_TR(warp == 0, r, 17);
            // S^T -> bf16 operand (and fp32 out after the last chunk)
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL], r & 1, abort_flag))) break;
            DN_TR(warp == 0, r, 18);
            tc_fence_after();
            {
                uint32_t v[64];
                tmem_ld64(tmem + lane_base + TM_S + 64 * h, v);
                st_row_bf16<64>(Sbf + h * 16384, d, 0, v);
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&bars[B_SBF]);
                DN_TR(warp == 0, r, 19);
                if (r == nch - 1 && x_out) {
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        x_out[(int64_t)(64 * h + c) * D + d] = __uint_as_float(v[c]);
                }
            }
            // O^T -> out (rows = tokens), two d_v columns per 4-byte store
            if (HAS_Q) {
                if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_OFULL], r & 1, abort_flag))) break;
                DN_TR(warp == 0, r, 20);
                tc_fence_after();
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + TM_O + 32 * h, v);
                tc_fence_before();
                mbar_arrive(&bars[B_OFREE]);
                DN_TR(warp == 0, r, 21);
                const int t0 = it.tok0 + r * kChunk + 32 * h;
                const int pc = d & ~1;
#pragma unroll
                for (int tt = 0; tt < 32; tt += 2) {
                    const float v0 = __uint_as_float(v[tt]), v1 = __uint_as_float(v[tt + 1]);
                    const float send = (lane & 1) ? v0 : v1;
                    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                    const int tok = t0 + tt + (lane & 1);
                    const uint32_t pk = (lane & 1) ? pack_bf16(recv, v1) : pack_bf16(v0, recv);
                    if (tok < it.tok1)
                        *reinterpret_cast<uint32_t*>(og + (int64_t)tok * p.o_st + pc) = pk;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kChainMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicExch(p.err, kErrTimeout);
}

}  // namespace tc
}  // namespace dn
