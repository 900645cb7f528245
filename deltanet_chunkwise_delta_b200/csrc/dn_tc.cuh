// Tensor-core (tcgen05 / TMEM / TMA) chain kernel for bf16, d_k = d_v = 128.
//
// Same per-chunk algorithm as dn_chain.cuh ("Linear Attention, Visualized",
// DeltaNet, "Complete per-chunk algorithm"), evaluated in the transposed
// domain so that every tensor-core product has M = 128:
//   T   = (I + B L)^{-1} B,  P = (Q K^T) o M_c   (from the UT pre-pass, dn_prep.cuh)
//   W^T = K^T T^T,  U^T = V^T T^T
//   Z^T = U^T - S^T W^T                  (accumulated into U^T's columns)
//   O^T = S^T Q^T + Z^T P^T
//   S^T <- S^T + Z^T K
// S^T (d_v lanes x d_k columns, fp32) lives in tensor memory for the whole run.
// Its bf16 copy, and that of Z^T, also live in tensor memory, where the
// products read them as their A operand: the state chain never goes through
// shared memory, which the products' B operands, the TMA loads and the
// epilogues share.
//
// Warp roles (512 threads):
//   warps 0-7   chain epilogue: Z^T -> bf16, S^T -> bf16 (tensor memory to
//               tensor memory), final state
//   warps 8-11  chunk-parallel epilogue: W^T -> bf16 rows in shared memory;
//               O -> global; lane 0 of warp 8 copies each chunk's P tile in
//   warp 12     issues the two state-chain products (Z^T, S^T update), one
//               thread; owns the tensor-memory allocation
//   warp 13     TMA loads of q, k (3-stage ring), one thread
//   warp 14     issues the chunk-parallel products (O^T, U^T, W^T), one thread
//   warp 15     TMA loads of v and bulk copies of T (2-stage ring), one thread
// The tensor pipe runs products in issue order, and a waiting issuer thread
// pays about 150 cycles per barrier even when the phase is already complete.
// So the chain issuer waits only for what the chain needs, and the parallel
// issuer, having done its own waits ahead of time, issues only inside the
// chain's two epilogue gaps (signalled by GAP1 / GAP2), where its products
// overlap the epilogues instead of delaying the next chain product.  Every
// wait on an mbarrier is bounded; on time-out the CTA drains, frees its
// tensor memory and reports DN_ERR_TIMEOUT through the error flag.
#pragma once

#include "dn_common.cuh"
#include "dn_sm100.cuh"

namespace dn {
namespace tc {

using namespace sm100;

constexpr int D = 128;
constexpr int kThreadsTc = 512;
constexpr int kMmaWarp = 12;
constexpr int kTmaWarp = 13;
constexpr int kParMmaWarp = 14;
constexpr int kTmaBWarp = 15;

// shared memory (byte offsets from a 1024-aligned base)
//   ring A (q, k): 3 stages of [Q d0-63 | K d0-63 | Q d64-127 | K d64-127]
//   ring B (v, T): 2 stages of [V d0-63 | V d64-127 | T]
//   O staging: 2 buffers of two 64-column boxes of token rows
constexpr int NA = 3, NB = 2;
constexpr int A_STAGE = 32768;
constexpr int OFF_B = NA * A_STAGE;
constexpr int B_STAGE = 24576, B_T = 16384;
constexpr int OFF_WB = OFF_B + NB * B_STAGE;   // W^T rows (d_k rows of 64 tokens)
constexpr int OFF_PB = OFF_WB + 16384;         // P rows
constexpr int OFF_OB = OFF_PB + 8192;          // O staging, 2 x 16 KB
constexpr int OFF_BAR = OFF_OB + 2 * 16384;
constexpr int NBAR = 31;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM_USED = OFF_MISC + 64;
constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// tensor-memory columns (512 allocated): S^T fp32, O^T, 2 x U^T/Z^T, W^T,
// Z^T bf16 (64 tokens in 32 columns), S^T bf16 (128 d_k in 64 columns)
constexpr uint32_t TM_S = 0, TM_O = 128, TM_ZU = 192, TM_WT = 320, TM_ZBF = 384, TM_SBF = 448;

// Barriers of a ring or of a double buffer come one per slot; a waiter on slot
// s for chunk r waits for that slot's (r / slots)-th completion.  Barriers
// completed by epilogue warps take one arrival per warp, after __syncwarp():
// each lane has already fenced its own writes or tensor-memory accesses.
enum : int {
    B_FULLA = 0,     // +3: q, k of a stage landed
    B_EMPTYA = 3,    // +3: stage of ring A consumed by both issuers
    B_FULLB = 6,     // +2: v, T landed
    B_EMPTYB = 8,    // +2: stage of ring B consumed
    B_WUFULL = 10,   // +2: W^T, U^T of the chunk ready in tensor memory
    B_WTFREE = 12,   // W^T columns read out
    B_WFULL = 13,    // W^T rows written to shared memory
    B_C1A = 14,      // Z^T = U^T - S^T W^T complete
    B_ZFULL = 15,    // bf16 Z^T written
    B_ZFREE = 16,    // +2: fp32 U^T / Z^T columns read out
    B_SFULL = 18,    // S^T updated
    B_SBF = 19,      // bf16 S^T written
    B_OFULL = 20,    // O^T complete
    B_OFREE = 21,    // O^T read out
    B_SBFREE = 22,   // O^T = S^T Q^T complete (bf16 S^T may be overwritten)
    B_PFULL = 23,    // P tile copied into shared memory
    B_GAP1 = 24,     // +2: chain issuer: Z^T of the chunk issued (one per chunk parity)
    B_GAP2 = 26,     // +2: chain issuer: S^T update of the chunk issued (one per chunk parity)
    B_OSTAGED = 28,  // O tile of the chunk staged as token rows
};
static_assert(B_OSTAGED < NBAR, "barrier count");

// Optional timeline of CTA 0 (build with -DDN_TRACE): globaltimer stamps per
// chunk and pipeline event, read back with dn_trace_copy().
#ifdef DN_TRACE
static __device__ unsigned long long g_dn_trace[64 * 32];
#define DN_TR(cond, r, slot)                                                                      \
    do {                                                                                          \
        if ((cond) && blockIdx.x == 0 && (r) >= 0 && (r) < 64 && (threadIdx.x & 31) == 0)          \
            g_dn_trace[(r) * 32 + (slot)] = globaltimer();                                        \
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

// N fp32 values -> N / 2 packed bf16 pairs (the tensor-memory A-operand layout).
template <int N>
__device__ __forceinline__ void pack_pairs(const uint32_t* v, uint32_t* out) {
#pragma unroll
    for (int c = 0; c < N / 2; ++c) out[c] = pack_bf16(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1]));
}

template <bool HAS_Q>
__global__ void __launch_bounds__(kThreadsTc, 1)
    k_tc_chain(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to, Params p) {
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
            mbar_init(&bars[B_ZFREE + s], 8);
        }
        mbar_init(&bars[B_WTFREE], 4);
        mbar_init(&bars[B_WFULL], 4);
        mbar_init(&bars[B_C1A], 1);
        mbar_init(&bars[B_ZFULL], 8);
        mbar_init(&bars[B_SFULL], 1);
        mbar_init(&bars[B_SBF], 8);
        mbar_init(&bars[B_OFULL], 1);
        mbar_init(&bars[B_OFREE], 4);
        mbar_init(&bars[B_SBFREE], 1);
        mbar_init(&bars[B_PFULL], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[B_GAP1 + s], 1);
            mbar_init(&bars[B_GAP2 + s], 1);
        }
        mbar_init(&bars[B_OSTAGED], 4);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kMmaWarp) {
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
            // the last loads issued must have landed before the CTA may exit (even after an abort)
            volatile int drain = 0;
            for (int r = issued - NA < 0 ? 0 : issued - NA; r < issued; ++r)
                mbar_wait(&bars[B_FULLA + (r % NA)], (r / NA) & 1, &drain, 200000000ull);
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
                bulk_load(st + B_T, p.wsT + ((size_t)(it.cbase + r) * p.sched.H + it.head) * kUnitBytes, 8192,
                          &bars[B_FULLB + s]);
                issued = r + 1;
            }
            volatile int drain = 0;
            for (int r = issued - 2 < 0 ? 0 : issued - 2; r < issued; ++r)
                mbar_wait(&bars[B_FULLB + (r & 1)], (r >> 1) & 1, &drain, 200000000ull);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ state-chain products
        // Only the two products on the chain: it waits for nothing else, and after
        // each one opens a gap for the chunk-parallel issuer.
        if (lane == 0 && nch > 0) {
            const uint32_t sb = saddr(smem);
            const uint32_t i_c1a = idesc_bf16(128, 64, false, true, true);
            const uint32_t i_c3 = idesc_bf16(128, 128, false, true);
            const uint64_t dW = sdesc(sb + OFF_WB, 8192, 1024);  // W^T rows, MN-major
            const uint64_t dK = sdesc(sb + 8192, 16384, 1024);   // K, MN-major
            for (int r = 0; r < nch; ++r) {
                const int sa = r % NA, s = r & 1;
                const uint64_t sta = (uint64_t)((sa * A_STAGE) >> 4);
                DN_TR(true, r, 0);
                if (!mbar_wait2(&bars[B_WFULL], r & 1, &bars[B_SBF], r & 1, abort_flag)) break;
                DN_TR(true, r, 3);
                tc_fence_after();
                // Z^T = U^T - S^T W^T
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    umma_bf16_ts(tmem + TM_ZU + s * 64, tmem + TM_SBF + 8 * j, dW + (uint64_t)((j * 2048) >> 4),
                                 i_c1a, has_v ? 1u : (j > 0 ? 1u : 0u));
                umma_commit(&bars[B_C1A]);
                mbar_arrive(&bars[B_GAP1 + s]);
                DN_TR(true, r, 1);
                if (!mbar_wait(&bars[B_ZFULL], r & 1, abort_flag)) break;
                DN_TR(true, r, 10);
                tc_fence_after();
                // S^T += Z^T K
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    umma_bf16_ts(tmem + TM_S, tmem + TM_ZBF + 8 * j, dK + sta + (uint64_t)((j * 2048) >> 4), i_c3,
                                 1u);
                umma_commit(&bars[B_SFULL]);
                umma_commit(&bars[B_EMPTYA + sa]);
                // gap barriers come one per chunk parity: the chain cannot get two chunks
                // ahead of the parallel issuer (Z^T of chunk r + 2 needs W^T of chunk r + 2,
                // which the parallel issuer issues after taking both gaps of chunk r), so
                // a waiter never misses a phase
                mbar_arrive(&bars[B_GAP2 + s]);
                DN_TR(true, r, 11);
            }
        }
    } else if (warp == kParMmaWarp) {
        // ------------------------------------------------------------ chunk-parallel products
        // Everything off the chain, issued only inside the chain's two gaps so that
        // it never queues in front of a chain product in the tensor pipe, and two
        // chunks ahead where it feeds the chain:
        //   gap 1 (after Z^T(r) is issued):  O^T = S^T Q^T of chunk r, U^T of chunk r+2
        //   gap 2 (after S^T(r+1) is issued): O^T += Z^T P^T of chunk r, W^T of chunk r+2
        // All waits for data and free buffers are done before waiting for the gap.
        if (lane == 0 && nch > 0) {
            const uint32_t sb = saddr(smem);
            const uint32_t i_tt = idesc_bf16(128, 64, true, false);
            const uint32_t i_o = idesc_bf16(128, 64, false, false);
            const uint64_t dKT = sdesc(sb + 8192, 16384, 1024);        // K^T, MN-major
            const uint64_t dVT = sdesc(sb + OFF_B, 8192, 1024);        // V^T, MN-major
            const uint64_t dT = sdesc(sb + OFF_B + B_T, 16, 1024);     // T^T, K-major
            const uint64_t dQ = sdesc(sb, 16, 1024);                   // Q^T, K-major
            const uint64_t dP = sdesc(sb + OFF_PB, 16, 1024);          // P^T, K-major
            // U^T of chunk c into its U^T / Z^T columns, once its v/T landed and the
            // columns' previous Z^T (chunk c - 2) is read out; W^T of chunk c once its
            // q/k and v/T landed and the previous W^T (chunk c - 1) is read out.  WUFULL
            // of the chunk is committed after its second product, EMPTYB after both.
            auto issue_u = [&](int c) -> bool {
                const int s = c & 1;
                if (!mbar_wait(&bars[B_FULLB + s], (c >> 1) & 1, abort_flag)) return false;
                if (c >= 2 && !mbar_wait(&bars[B_ZFREE + s], ((c >> 1) - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                if (has_v) {
                    const uint64_t stb = (uint64_t)((s * B_STAGE) >> 4);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_bf16(tmem + TM_ZU + s * 64, dVT + stb + (uint64_t)((j * 2048) >> 4),
                                  dT + stb + (uint64_t)((j * 32) >> 4), i_tt, j > 0);
                }
                return true;
            };
            auto issue_w = [&](int c) -> bool {
                const int sa = c % NA, s = c & 1;
                if (!mbar_wait2(&bars[B_FULLA + sa], (c / NA) & 1, &bars[B_FULLB + s], (c >> 1) & 1, abort_flag))
                    return false;
                if (c >= 1 && !mbar_wait(&bars[B_WTFREE], (c - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint64_t sta = (uint64_t)((sa * A_STAGE) >> 4);
                const uint64_t stb = (uint64_t)((s * B_STAGE) >> 4);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    umma_bf16(tmem + TM_WT, dKT + sta + (uint64_t)((j * 2048) >> 4),
                              dT + stb + (uint64_t)((j * 32) >> 4), i_tt, j > 0);
                umma_commit(&bars[B_WUFULL + s]);
                umma_commit(&bars[B_EMPTYB + s]);
                return true;
            };
            // chunks 0 and 1 before the chain starts (W^T of chunk 1 waits until the
            // epilogue has read chunk 0's)
            bool ok = issue_u(0) && issue_w(0);
            if (ok && nch > 1) ok = issue_u(1) && issue_w(1);
            for (int r = 0; ok && r < nch; ++r) {
                const int sa = r % NA;
                const uint64_t sta = (uint64_t)((sa * A_STAGE) >> 4);
                const bool ahead = r + 2 < nch;
                // ---- gap 1
                if (HAS_Q && !mbar_wait(&bars[B_OFREE], r & 1, abort_flag)) break;
                if (!mbar_wait(&bars[B_GAP1 + (r & 1)], (r >> 1) & 1, abort_flag)) break;
                DN_TR(true, r, 6);
                tc_fence_after();
                if (HAS_Q) {
                    // O^T = S^T Q^T
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint64_t o = (uint64_t)(((j >> 2) * 16384 + (j & 3) * 32) >> 4);
                        umma_bf16_ts(tmem + TM_O, tmem + TM_SBF + 8 * j, dQ + sta + o, i_o, j > 0);
                    }
                    umma_commit(&bars[B_SBFREE]);
                }
                umma_commit(&bars[B_EMPTYA + sa]);
                if (ahead && !issue_u(r + 2)) break;
                DN_TR(true, r, 7);
                // ---- gap 2
                if (HAS_Q && !mbar_wait(&bars[B_PFULL], r & 1, abort_flag)) break;
                if (!mbar_wait(&bars[B_GAP2 + (r & 1)], (r >> 1) & 1, abort_flag)) break;
                DN_TR(true, r, 12);
                tc_fence_after();
                if (HAS_Q) {
                    // O^T += Z^T P^T
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_bf16_ts(tmem + TM_O, tmem + TM_ZBF + 8 * j, dP + (uint64_t)((j * 32) >> 4), i_o, 1u);
                    umma_commit(&bars[B_OFULL]);
                }
                if (ahead && !issue_w(r + 2)) break;
                DN_TR(true, r, 4);
            }
        }
    } else if (warp >= 8 && warp < 12) {
        // ------------------------------------------------------------ chunk-parallel epilogue
        const int q = warp - 8;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        int p_issued = 0;
        // P tile of chunk c into its buffer (one thread)
        auto issue_p = [&](int c) {
            ++p_issued;
            mbar_expect_tx(&bars[B_PFULL], 8192u);
            bulk_load(smem + OFF_PB, p.wsT + ((size_t)(it.cbase + c) * p.sched.H + it.head) * kUnitBytes + 8192,
                      8192, &bars[B_PFULL]);
        };
        // O^T of chunk c -> out.  Each lane holds one d_v row of O^T (64 tokens), so the
        // tile is staged as token rows (two boxes of 64 columns, 128-byte swizzled rows,
        // the TMA box layout of out) and written out by one TMA store per box; a chunk
        // that ends inside the run's last 64 tokens is written with bounded 16-byte
        // stores instead.  Two staging buffers: a warp staging chunk c + 2 has passed
        // OSTAGED(c + 1), to which every warp arrives only after it (and, for warp 8,
        // the TMA store it issued) has finished reading chunk c.
        __nv_bfloat16* og = static_cast<__nv_bfloat16*>(p.o) + it.b * p.o_sb + it.head * p.o_sh;
        const int d = 32 * q + lane;
        auto store_o = [&](int c) -> bool {
            tc_fence_after();
            uint32_t v[64];
            tmem_ld64(tmem + lane_base + TM_O, v);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_OFREE]);
            DN_TR(q == 0, c, 21);
            uint8_t* ob = smem + OFF_OB + (c & 1) * 16384;
            __nv_bfloat16* box = reinterpret_cast<__nv_bfloat16*>(ob + (d >> 6) * 8192);
#pragma unroll
            for (int t = 0; t < 64; ++t)
                box[swz128(t, d & 63) >> 1] = __float2bfloat16_rn(__uint_as_float(v[t]));
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_OSTAGED]);
            DN_TR(q == 0, c, 28);
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_OSTAGED], c & 1, abort_flag))) return false;
            const int t0 = it.tok0 + c * kChunk;
            if (t0 + kChunk <= it.tok1) {
                if (q == 0 && lane == 0) {
                    tma_store_4d(&to, ob, 0, it.head, t0, it.b);
                    tma_store_4d(&to, ob + 8192, 64, it.head, t0, it.b);
                    bulk_commit();
                    bulk_wait_read0();
                }
                __syncwarp();
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int id = 32 * q + lane + 128 * k, t = id >> 4, dc = id & 15;
                    const uint4 row = *reinterpret_cast<const uint4*>(ob + (dc >> 3) * 8192 + swz128(t, (dc & 7) * 8));
                    if (t0 + t < it.tok1) *reinterpret_cast<uint4*>(og + (int64_t)(t0 + t) * p.o_st + 8 * dc) = row;
                }
            }
            DN_TR(q == 0, c, 26);
            return true;
        };
        if (HAS_Q && lane == 0) mbar_arrive(&bars[B_OFREE]);
        for (int r = 0; r < nch; ++r) {
            const int s = r & 1;
            // W^T (tensor memory, d_k lanes) -> bf16 rows of 64 tokens (an MN-major
            // operand), once the previous rows are consumed
            if (r >= 1 && !__all_sync(0xffffffffu, mbar_wait(&bars[B_C1A], (r - 1) & 1, abort_flag))) break;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_WUFULL + s], (r >> 1) & 1, abort_flag))) break;
            DN_TR(q == 0, r, 13);
            tc_fence_after();
            {
                uint32_t v[64];
                tmem_ld64(tmem + lane_base + TM_WT, v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_WTFREE]);
                st_row_bf16<64>(Wb, 32 * q + lane, 0, v);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_WFULL]);
            DN_TR(q == 0, r, 14);
            if (HAS_Q && r >= 1) {
                // chunk r - 1 complete: copy in chunk r's P tile, write out O of chunk r - 1
                if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_OFULL], (r - 1) & 1, abort_flag))) break;
                if (q == 0 && lane == 0) issue_p(r);
                if (!store_o(r - 1)) break;
            } else if (HAS_Q && q == 0 && lane == 0) {
                issue_p(0);
            }
        }
        if (HAS_Q && nch > 0 && !*abort_flag &&
            __all_sync(0xffffffffu, mbar_wait(&bars[B_OFULL], (nch - 1) & 1, abort_flag)))
            store_o(nch - 1);
        // the last P copy must have landed, and the TMA stores of O completed, before
        // the CTA may exit (even after an abort)
        if (lane == 0 && p_issued > 0) {
            volatile int drain = 0;
            mbar_wait(&bars[B_PFULL], (p_issued - 1) & 1, &drain, 200000000ull);
        }
        if (HAS_Q && q == 0 && lane == 0) bulk_wait0();
    } else if (warp < 8) {
        // ------------------------------------------------------------ chain epilogue
        // Warp w handles d_v rows 32 (w % 4) .. + 31 (its tensor-memory lane quarter)
        // and half h = w / 4 of the columns.
        const int wq = warp & 3, h = warp >> 2;
        const int d = 32 * wq + lane;  // d_v row of S^T, Z^T
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
                uint32_t pk[32];
                pack_pairs<64>(v, pk);
                tmem_st32(tmem + lane_base + TM_SBF + 32 * h, pk);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_SBF]);
        for (int r = 0; r < nch; ++r) {
            const int s = r & 1;
            // Z^T -> bf16 (A operand of the S^T update and of O^T += Z^T P^T), once the
            // previous chunk's O^T += Z^T P^T has read the previous one
            DN_TR(warp == 0, r, 27);
            if (HAS_Q && r >= 1 &&
                !__all_sync(0xffffffffu, mbar_wait(&bars[B_OFULL], (r - 1) & 1, abort_flag)))
                break;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_C1A], r & 1, abort_flag))) break;
            DN_TR(warp == 0, r, 16);
            tc_fence_after();
            {
                uint32_t v[32], pk[16];
                tmem_ld32(tmem + lane_base + TM_ZU + s * 64 + 32 * h, v);
                pack_pairs<32>(v, pk);
                tmem_st16(tmem + lane_base + TM_ZBF + 16 * h, pk);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_ZFULL]);
                mbar_arrive(&bars[B_ZFREE + s]);
            }
            DN_TR(warp == 0, r, 17);
            // S^T -> bf16 (and fp32 out after the last chunk), once S^T Q^T has read the
            // previous bf16 copy
            if (HAS_Q && !__all_sync(0xffffffffu, mbar_wait(&bars[B_SBFREE], r & 1, abort_flag))) break;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL], r & 1, abort_flag))) break;
            DN_TR(warp == 0, r, 18);
            tc_fence_after();
            {
                uint32_t v[64], pk[32];
                tmem_ld64(tmem + lane_base + TM_S + 64 * h, v);
                pack_pairs<64>(v, pk);
                tmem_st32(tmem + lane_base + TM_SBF + 32 * h, pk);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_SBF]);
                DN_TR(warp == 0, r, 19);
                if (r == nch - 1 && x_out) {
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        x_out[(int64_t)(64 * h + c) * D + d] = __uint_as_float(v[c]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicExch(p.err, kErrTimeout);
}

}  // namespace tc
}  // namespace dn
