// Tensor-core summary pass of the context-parallel split (bf16, d_k = d_v = 128).
//
// "Context Parallelism for DeltaNet", section 3: the chunk update is affine in
// the incoming state, S_out = S_in P_g + H_g over a run g of chunks, so runs
// compose.  Each item of this kernel is one run of one (sequence, head):
//   run 0     (E):  the run's end state from the true initial state
//   run g >= 1 (HP): both maps of the run at once:
//                    H_g  the run's end state from a zero start (values V),
//                    P_g  the product of the chunk transitions (start I, no values).
// Both chains are the per-chunk recurrence of dn_tc.cuh without outputs, in the
// transposed domain (every product M = 128):
//   W^T = K^T T^T, U^T = V^T T^T                     (chunk-parallel, shared)
//   Z_H^T = U^T + S_H^T (-W^T),  Z_P^T = S_P^T (-W^T) (one product per chain)
//   S_x^T <- S_x^T + Z_x^T K                          (one product per chain)
// The two chains share the loads of k, v and T, the W^T product and its -W
// rows, and run interleaved on the tensor pipe: chain P's products fill the gaps
// of chain H's epilogues and the other way round.  S_x^T (fp32) lives in tensor
// memory; the bf16 copy that the first product reads as its A operand is in
// tensor memory for chain H and in shared memory for chain P (which frees the
// columns W^T of the next chunk is formed in while the chain runs); Z_x^T in
// bf16 goes to shared memory (the A operand of the state update).
//
// Warp roles (512 threads):
//   warps 0-3   chain H epilogue (lane quarter w, all columns)
//   warps 4-7   chain P epilogue (idle for E items)
//   warps 8-11  W^T -> -W token rows in the chunk's k stage
//   warp 12     issues the chain products, one thread; owns the tensor memory
//   warp 13     TMA loads of k (3-stage ring), one thread
//   warp 14     issues W^T of the next chunk once the chunk's first products
//               are queued, and U^T once chain H's state update is, one thread
//   warp 15     TMA loads of v and bulk copies of T (2-stage ring), one thread
// Every wait on an mbarrier is bounded; on time-out the CTA drains, frees its
// tensor memory and reports DN_ERR_TIMEOUT through the error flag.
#pragma once

#include <type_traits>

#include "dn_common.cuh"
#include "dn_sm100.cuh"
#include "dn_tc.cuh"

namespace dn {
namespace tcs {

using namespace sm100;
using tc::D;
using tc::pack_pairs;
using tc::RowFrags;
using tc::store_token_rows;
using tc::tmem_load_rows;

constexpr int kThreadsSum = 512;
constexpr int kMmaWarp = 12;
constexpr int kTmaWarp = 13;
constexpr int kParMmaWarp = 14;
constexpr int kTmaBWarp = 15;

// shared memory (byte offsets from a 1024-aligned base)
//   ring A: 3 stages of [-W d0-63 | -W d64-127 | K d0-63 | K d64-127] (-W rows
//           written by the epilogue, k by TMA)
//   ring B: 2 stages of [V d0-63 | V d64-127 | T]
//   Z^T bf16 of chain H and of chain P: d_v rows x 64 tokens, 128-byte swizzled
//   S_P^T bf16: d_v rows x [d_k 0-63 | d_k 64-127], 128-byte swizzled
//   (Gated DeltaNet: ring B stages also hold T' = T diag(lambda[1:l]), the W<- factor, and a
//   2-slot ring holds each chunk's row factors from the pre-pass: lambda[l+1:C] per row,
//   which scales Z^T's token columns (Z^T diag(lambda[l+1:C]) K = Z^T K->), and lambda[1:C])
constexpr int NA = 3, NB = 2;
constexpr int A_STAGE = 32768;
constexpr int A_K = 16384;
constexpr int OFF_B = NA * A_STAGE;
constexpr int B_T = 16384, B_T2 = 24576;
constexpr int Z_BYTES = 16384;
constexpr int NF = 2;  // Gated DeltaNet: slots of the row-factor ring
constexpr int NBAR = 31;
template <bool GATED>
struct SumLay {
    static constexpr int B_STAGE = GATED ? 32768 : 24576;
    static constexpr int OFF_Z = OFF_B + NB * B_STAGE;
    static constexpr int OFF_SP = OFF_Z + 2 * Z_BYTES;
    static constexpr int OFF_F = OFF_SP + 32768;  // row-factor ring (gated)
    static constexpr int OFF_BAR = OFF_F + (GATED ? NF * kUnitFBytes : 0);
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM_USED = OFF_MISC + 64;
    static constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
};
static_assert(SumLay<false>::SMEM_BYTES <= 232448 && SumLay<true>::SMEM_BYTES <= 232448, "shared memory budget");
constexpr int SMEM_BYTES = SumLay<false>::SMEM_BYTES;

// 32 consecutive 32-bit tensor-memory columns of this thread's lane, without
// waiting: follow with tmem_wait_st() before the columns are signalled as written.
__device__ __forceinline__ void tmem_st32_nowait(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// tensor-memory columns (512 allocated), chain x = 0 (H) or 1 (P): S_x^T fp32,
// U^T / Z_H^T and Z_P^T fp32 (64 tokens), S_H^T bf16 (128 d_k in 64 columns), W^T
__device__ __forceinline__ uint32_t tm_s(int x) { return 128u * (uint32_t)x; }
__device__ __forceinline__ uint32_t tm_zu(int x) { return 256u + 64u * (uint32_t)x; }
constexpr uint32_t TM_SBF = 384, TM_WT = 448;

// Barriers: one per slot for rings, one per chain for the chain's own steps.
enum : int {
    B_FULLA = 0,    // +3: k of a stage landed
    B_EMPTYA = 3,   // +3: stage of ring A consumed
    B_FULLB = 6,    // +2: v, T landed
    B_EMPTYB = 8,   // +2: stage of ring B consumed
    B_WUFULL = 10,  // W^T of the chunk complete
    B_WFULL = 11,   // -W rows of the chunk written to its ring-A stage (W^T read out)
    B_UFULL = 12,   // U^T of the chunk complete (in chain H's Z columns)
    B_C1 = 13,      // +2: Z_x^T product complete
    B_ZFULL = 15,   // +2: Z_x^T written (bf16, shared memory) and its fp32 columns read out
    B_SFULL = 17,   // +2: S_x^T updated
    B_SBF = 19,     // +2: bf16 S_x^T written
    B_GAP1 = 21,    // +2: the chunk's first products are issued (one per chunk parity)
    B_GAP2 = 23,    // +2: chain H's state update is issued (one per chunk parity)
    B_DRAIN = 25,   // +2: drain of the chain issuer's / the parallel issuer's products
    B_FULLF = 27,   // +2: row factors of a chunk landed (gated)
    B_EMPTYF = 29,  // +2: row-factor slot read by every chain-epilogue warp (gated)
};
static_assert(B_EMPTYF + NF <= NBAR, "barrier count");

// Optional timeline of CTA 1 (the first two-chain item of a split chain; build
// with -DDN_TRACE): globaltimer stamps per chunk and pipeline event.
#ifdef DN_TRACE
static __device__ unsigned long long g_dn_trace_sum[64 * 32];
#define DN_TS(cond, r, slot)                                                                      \
    do {                                                                                          \
        if ((cond) && blockIdx.x == 1 && (r) >= 0 && (r) < 64 && (threadIdx.x & 31) == 0)          \
            g_dn_trace_sum[(r) * 32 + (slot)] = globaltimer();                                    \
    } while (0)
#else
#define DN_TS(cond, r, slot) \
    do {                     \
    } while (0)
#endif

template <bool GATED>
static __global__ void __launch_bounds__(kThreadsSum, 1)
    k_tc_summary(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv, Params p) {
    using L = SumLay<GATED>;
    constexpr int kUnit = unit_bytes(GATED);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int n_items = count_A(p.sched);
    if ((int)blockIdx.x >= n_items) return;
    int mode = kModeEnd;
    const Item it = item_A(p.sched, blockIdx.x, mode);

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    WaitCtl* ctl = reinterpret_cast<WaitCtl*>(smem + L::OFF_MISC + 8);
    volatile int* abort_flag = &ctl->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NA; ++s) {
            mbar_init(&bars[B_FULLA + s], 1);
            mbar_init(&bars[B_EMPTYA + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[B_FULLB + s], 1);
            mbar_init(&bars[B_EMPTYB + s], 1);
            mbar_init(&bars[B_C1 + s], 1);
            mbar_init(&bars[B_ZFULL + s], 4);
            mbar_init(&bars[B_SFULL + s], 1);
            mbar_init(&bars[B_SBF + s], 4);
            mbar_init(&bars[B_GAP1 + s], 1);
            mbar_init(&bars[B_GAP2 + s], 1);
        }
        mbar_init(&bars[B_WUFULL], 1);
        mbar_init(&bars[B_WFULL], 4);
        mbar_init(&bars[B_UFULL], 1);
        mbar_init(&bars[B_DRAIN], 1);
        mbar_init(&bars[B_DRAIN + 1], 1);
        for (int s = 0; s < NF; ++s) {
            mbar_init(&bars[B_FULLF + s], 1);
            mbar_init(&bars[B_EMPTYF + s], mode == kModeHP ? 8 : 4);
        }
        wait_ctl_init(ctl, p.wait_ns);
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

    // the item's chain count is a compile-time constant of the role code below, so
    // that each issuing thread runs straight-line product sequences
    auto roles = [&](auto two_c) {
        constexpr bool TWO = decltype(two_c)::value;
        if (warp == kTmaWarp) {
            // ------------------------------------------------------------ ring A: k
            if (lane == 0 && nch > 0) {
                int issued = 0;
                for (int r = 0; r < nch; ++r) {
                    const int s = r % NA;
                    if (r >= NA && !mbar_wait(&bars[B_EMPTYA + s], ((r / NA) - 1) & 1, abort_flag)) break;
                    mbar_expect_tx(&bars[B_FULLA + s], 16384u);
                    uint8_t* st = smem + s * A_STAGE;
                    const int t0 = it.tok0 + r * kChunk;
    #pragma unroll
                    for (int a = 0; a < 2; ++a)
                        tma_load_4d(st + A_K + a * 8192, &tk, &bars[B_FULLA + s], a * 64, it.head, t0, it.b);
                    issued = r + 1;
                }
                // the last loads issued must have landed before the CTA may exit (even after an abort)
                volatile int drain = 0;
                for (int r = issued - NA < 0 ? 0 : issued - NA; r < issued; ++r)
                    mbar_wait(&bars[B_FULLA + (r % NA)], (r / NA) & 1, &drain, kDrainWaitNs);
            }
        } else if (warp == kTmaBWarp) {
            // ------------------------------------------------------------ ring B: v, T
            if (lane == 0 && nch > 0) {
                int issued = 0, f_issued = 0;
                for (int r = 0; r < nch; ++r) {
                    const int s = r & 1;
                    if (r >= 2 && !mbar_wait(&bars[B_EMPTYB + s], ((r >> 1) - 1) & 1, abort_flag)) break;
                    mbar_expect_tx(&bars[B_FULLB + s], 16384u + 8192u + (GATED ? 8192u : 0u));
                    uint8_t* st = smem + OFF_B + s * L::B_STAGE;
                    const int t0 = it.tok0 + r * kChunk;
    #pragma unroll
                    for (int a = 0; a < 2; ++a) tma_load_4d(st + a * 8192, &tv, &bars[B_FULLB + s], a * 64, it.head, t0, it.b);
                    const uint8_t* unit = p.wsT + ((size_t)(it.cbase + r) * p.sched.H + it.head) * kUnit;
                    bulk_load(st + B_T, unit, 8192, &bars[B_FULLB + s]);
                    issued = r + 1;
                    if constexpr (GATED) {
                        bulk_load(st + B_T2, unit + kUnitT2, 8192, &bars[B_FULLB + s]);
                        // the chunk's row factors, once the chain epilogues are done with
                        // chunk r - 2's
                        const int sf = r % NF;
                        if (r >= NF && !mbar_wait(&bars[B_EMPTYF + sf], ((r / NF) - 1) & 1, abort_flag)) break;
                        mbar_expect_tx(&bars[B_FULLF + sf], (uint32_t)kUnitFBytes);
                        bulk_load(smem + L::OFF_F + sf * kUnitFBytes, unit + kUnitF, kUnitFBytes, &bars[B_FULLF + sf]);
                        f_issued = r + 1;
                    }
                }
                volatile int drain = 0;
                for (int r = issued - 2 < 0 ? 0 : issued - 2; r < issued; ++r)
                    mbar_wait(&bars[B_FULLB + (r & 1)], (r >> 1) & 1, &drain, kDrainWaitNs);
                for (int r = f_issued - NF < 0 ? 0 : f_issued - NF; r < f_issued; ++r)
                    mbar_wait(&bars[B_FULLF + (r % NF)], (r / NF) & 1, &drain, kDrainWaitNs);
            }
        } else if (warp == kMmaWarp) {
            // ------------------------------------------------------------ chain products
            // Per chunk and chain: Z_x^T = [U^T] + S_x^T (-W^T), then S_x^T += Z_x^T K.
            // Chain P's first product is queued behind chain H's, and each state
            // update as soon as its chain's Z^T is in shared memory.  Gap 1 (after the
            // first products) lets the parallel issuer queue W^T of the next chunk, gap
            // 2 (after chain H's update) its U^T.
            if (lane == 0 && nch > 0) {
                const uint32_t sb = saddr(smem);
                const uint32_t i_c1 = idesc_bf16(128, 64, false, false);
                const uint32_t i_c3 = idesc_bf16(128, 128, false, true);
                const uint64_t dW = sdesc(sb, 16, 1024);             // -W token rows, K-major
                const uint64_t dK = sdesc(sb + A_K, 8192, 1024);     // K, MN-major
                const uint64_t dZ = sdesc(sb + L::OFF_Z, 16, 1024);     // Z^T rows, K-major (+ Z_BYTES for P)
                const uint64_t dSP = sdesc(sb + L::OFF_SP, 16, 1024);   // S_P^T bf16 rows, K-major
                for (int r = 0; r < nch; ++r) {
                    const int sa = r % NA;
                    const uint64_t sta = (uint64_t)((sa * A_STAGE) >> 4);
                    DN_TS(true, r, 0);
                    if (!mbar_wait3(&bars[B_WFULL], r & 1, &bars[B_SBF], r & 1, &bars[B_UFULL], r & 1, abort_flag))
                        break;
                    DN_TS(true, r, 1);
                    // chain H: Z_H^T = U^T + S_H^T (-W^T), A operand (bf16 S_H^T) in tensor memory
                    tc_fence_after();
    #pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint64_t o = (uint64_t)(((j >> 2) * 8192 + (j & 3) * 32) >> 4);
                        umma_bf16_ts(tmem + tm_zu(0), tmem + TM_SBF + 8 * j, dW + sta + o, i_c1, 1u);
                    }
                    umma_commit(&bars[B_C1]);
                    DN_TS(true, r, 2);
                    if constexpr (TWO) {
                        // chain P: Z_P^T = S_P^T (-W^T), A operand in shared memory
                        if (!mbar_wait(&bars[B_SBF + 1], r & 1, abort_flag)) break;
                        tc_fence_after();
    #pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const uint64_t o = (uint64_t)(((j >> 2) * 8192 + (j & 3) * 32) >> 4);
                            const uint64_t oa = (uint64_t)(((j >> 2) * 16384 + (j & 3) * 32) >> 4);
                            umma_bf16(tmem + tm_zu(1), dSP + oa, dW + sta + o, i_c1, j > 0 ? 1u : 0u);
                        }
                        umma_commit(&bars[B_C1 + 1]);
                        DN_TS(true, r, 3);
                    }
                    mbar_arrive(&bars[B_GAP1 + (r & 1)]);
                    // S_H^T += Z_H^T K
                    if (!mbar_wait(&bars[B_ZFULL], r & 1, abort_flag)) break;
                    DN_TS(true, r, 4);
                    tc_fence_after();
    #pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_bf16(tmem + tm_s(0), dZ + (uint64_t)((j * 32) >> 4), dK + sta + (uint64_t)((j * 2048) >> 4),
                                  i_c3, 1u);
                    umma_commit(&bars[B_SFULL]);
                    DN_TS(true, r, 5);
                    mbar_arrive(&bars[B_GAP2 + (r & 1)]);
                    if constexpr (TWO) {
                        // S_P^T += Z_P^T K
                        if (!mbar_wait(&bars[B_ZFULL + 1], r & 1, abort_flag)) break;
                        DN_TS(true, r, 6);
                        tc_fence_after();
                        const uint64_t zo = (uint64_t)(Z_BYTES >> 4);
    #pragma unroll
                        for (int j = 0; j < 4; ++j)
                            umma_bf16(tmem + tm_s(1), dZ + zo + (uint64_t)((j * 32) >> 4),
                                      dK + sta + (uint64_t)((j * 2048) >> 4), i_c3, 1u);
                        umma_commit(&bars[B_SFULL + 1]);
                        DN_TS(true, r, 7);
                    }
                    // the stage's -W rows and k are read by the products above (and k by W^T of
                    // the chunk, complete before its -W rows were written)
                    umma_commit(&bars[B_EMPTYA + sa]);
                }
                umma_drain(&bars[B_DRAIN]);
            }
        } else if (warp == kParMmaWarp) {
            // ------------------------------------------------------------ chunk-parallel products
            // W^T and U^T (into chain H's Z columns) of chunk r + 1, each issued in one of
            // the chain's gaps so that it never queues in front of a chain product: W^T
            // once chunk r's first products are queued (its own -W rows were read out
            // before them), U^T once Z_H^T(r) has been read out and chain H's update is
            // queued.
            if (lane == 0 && nch > 0) {
                const uint32_t sb = saddr(smem);
                const uint32_t i_tt = idesc_bf16(128, 64, true, false);
                const uint64_t dKT = sdesc(sb + A_K, 8192, 1024);          // K^T, MN-major
                const uint64_t dVT = sdesc(sb + OFF_B, 8192, 1024);        // V^T, MN-major
                const uint64_t dT = sdesc(sb + OFF_B + B_T, 16, 1024);     // T^T, K-major
                // W = T K, or for Gated DeltaNet W<- = T' K with T' = T diag(lambda[1:l])
                const uint64_t dTw = GATED ? sdesc(sb + OFF_B + B_T2, 16, 1024) : dT;
                auto issue_w = [&](int c) {
                    const uint64_t sta = (uint64_t)(((c % NA) * A_STAGE) >> 4);
                    const uint64_t stb = (uint64_t)(((c & 1) * L::B_STAGE) >> 4);
    #pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_bf16(tmem + TM_WT, dKT + sta + (uint64_t)((j * 2048) >> 4),
                                  dTw + stb + (uint64_t)((j * 32) >> 4), i_tt, j > 0);
                    umma_commit(&bars[B_WUFULL]);
                };
                // U^T of chunk c; its ring-B stage is consumed after it (W^T came first)
                auto issue_u = [&](int c) {
                    const int s = c & 1;
                    const uint64_t stb = (uint64_t)((s * L::B_STAGE) >> 4);
    #pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_bf16(tmem + tm_zu(0), dVT + stb + (uint64_t)((j * 2048) >> 4),
                                  dT + stb + (uint64_t)((j * 32) >> 4), i_tt, j > 0);
                    umma_commit(&bars[B_UFULL]);
                    umma_commit(&bars[B_EMPTYB + s]);
                };
                auto wait_data = [&](int c) -> bool {
                    return mbar_wait2(&bars[B_FULLA + c % NA], (c / NA) & 1, &bars[B_FULLB + (c & 1)], (c >> 1) & 1,
                                      abort_flag);
                };
                bool ok = wait_data(0);
                if (ok) {
                    tc_fence_after();
                    issue_w(0);
                    issue_u(0);
                }
                for (int r = 0; ok && r + 1 < nch; ++r) {
                    // gap 1: chunk r + 1's data; W^T(r) was read out before chunk r's products
                    if (!wait_data(r + 1) || !mbar_wait(&bars[B_GAP1 + (r & 1)], (r >> 1) & 1, abort_flag)) break;
                    DN_TS(true, r, 8);
                    tc_fence_after();
                    issue_w(r + 1);
                    // gap 2: Z_H^T(r) read out of the U^T columns, chain H's update queued
                    if (!mbar_wait(&bars[B_ZFULL], r & 1, abort_flag) ||
                        !mbar_wait(&bars[B_GAP2 + (r & 1)], (r >> 1) & 1, abort_flag))
                        break;
                    DN_TS(true, r, 9);
                    tc_fence_after();
                    issue_u(r + 1);
                }
                umma_drain(&bars[B_DRAIN + 1]);
            }
        } else if (warp >= 8 && warp < 12) {
            // ------------------------------------------------------------ -W rows
            const int q = warp - 8;
            const uint32_t lane_base = (uint32_t)(32 * q) << 16;
            for (int r = 0; r < nch; ++r) {
                uint8_t* stage = smem + (r % NA) * A_STAGE;
                // W^T (tensor memory, d_k lanes) -> -W token rows in the chunk's k stage,
                // once the stage holds the chunk (its previous chunk's products are done)
                if (!__all_sync(0xffffffffu, mbar_wait2(&bars[B_WUFULL], r & 1, &bars[B_FULLA + r % NA], (r / NA) & 1,
                                                        abort_flag)))
                    break;
                DN_TS(q == 0, r, 10);
                tc_fence_after();
                {
                    RowFrags f;
                    tmem_load_rows(tmem + lane_base + TM_WT, f);
                    tc_fence_before();
                    store_token_rows(f, q, stage, 8192, -1.f);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_WFULL]);
                DN_TS(q == 0, r, 11);
            }
        } else if (warp < 8) {
            // ------------------------------------------------------------ chain epilogues
            // Warp w serves chain x = w / 4 and d_v rows 32 (w % 4) .. + 31 (its lane quarter).
            const int x = warp >> 2, wq = warp & 3;
            const int d = 32 * wq + lane;  // d_v row of S_x^T, Z_x^T
            const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
            if (x == 0 || TWO) {
                // start state and destination of this chain
                const float* x_in = nullptr;
                float* x_out;
                if (x == 1) {
                    x_out = p.wsP + (int64_t)(it.slot + it.g) * D * D;
                } else if (mode == kModeEnd) {
                    x_in = p.s0 ? p.s0 + it.seq * p.s0_sn + it.head * p.s0_sh : nullptr;
                    x_out = p.wsH + (int64_t)it.slot * D * D;
                } else {
                    x_out = p.wsH + (int64_t)(it.slot + it.g) * D * D;
                }
                uint8_t* zs = smem + L::OFF_Z + x * Z_BYTES;
                // bf16 copy of S_x^T columns 64 hh .. + 63 of row d: chain H into tensor
                // memory, chain P into K block hh of its shared-memory operand
                auto store_sbf = [&](int xx, int hh, const uint32_t(&pk)[32]) {
                    if (xx == 0) {
                        tmem_st32_nowait(tmem + lane_base + TM_SBF + 32 * hh, pk);
                    } else {
                        uint8_t* sp = smem + L::OFF_SP + hh * 16384;
    #pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<uint4*>(sp + swz128(d, 8 * c)) =
                                make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                    }
                };
                // Gated DeltaNet: the row factors of chunk c (lambda[l+1:C] per row, then
                // lambda[1:C]), held from B_FULLF until this warp's Z^T of the chunk is converted
                auto ffac = [&](int c) {
                    return reinterpret_cast<const float*>(smem + L::OFF_F + (c % NF) * kUnitFBytes);
                };
                // the update of chunk 0 adds K->^T Z to lambda[1:C] S
                bool live = true;
                float lam0 = 1.f;
                if (GATED && nch > 0) {
                    live = __all_sync(0xffffffffu, mbar_wait(&bars[B_FULLF], 0, abort_flag));
                    if (live) lam0 = ffac(0)[kChunk];
                }
    #pragma unroll 1
                for (int hh = 0; live && hh < 2; ++hh) {
                    uint32_t v[64];
    #pragma unroll
                    for (int c = 0; c < 64; ++c) {
                        const int a = 64 * hh + c;
                        float y = 0.f;
                        if (x_in) y = x_in[(int64_t)a * D + d];
                        else if (x == 1) y = (a == d) ? 1.f : 0.f;
                        v[c] = __float_as_uint(y);
                    }
                    if (nch == 0) {
                        for (int c = 0; c < 64; ++c) x_out[(int64_t)(64 * hh + c) * D + d] = __uint_as_float(v[c]);
                    } else {
                        uint32_t pk[32];
                        pack_pairs<64>(v, pk);
                        store_sbf(x, hh, pk);
                        if constexpr (GATED) {
    #pragma unroll
                            for (int c = 0; c < 64; ++c) v[c] = __float_as_uint(lam0 * __uint_as_float(v[c]));
                        }
                        tmem_st32(tmem + lane_base + tm_s(x) + 64 * hh, *reinterpret_cast<uint32_t(*)[32]>(v));
                        tmem_st32(tmem + lane_base + tm_s(x) + 64 * hh + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                    }
                }
                tmem_wait_st();  // the bf16 copy's tensor-memory stores
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0 && live) mbar_arrive(&bars[B_SBF + x]);
                for (int r = 0; live && r < nch; ++r) {
                    // Z_x^T -> bf16 token columns of row d in shared memory (the A operand of
                    // the state update)
                    if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_C1 + x], r & 1, abort_flag))) break;
                    DN_TS(wq == 0, r, 12 + 4 * x);
                    tc_fence_after();
    #pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t v[32], pk[16];
                        tmem_ld32(tmem + lane_base + tm_zu(x) + 32 * hh, v);
                        if constexpr (GATED) {
                            // Z^T diag(lambda[l+1:C]): the update then adds K->^T Z
                            const float4* f4 = reinterpret_cast<const float4*>(ffac(r) + 32 * hh);
    #pragma unroll
                            for (int c4 = 0; c4 < 8; ++c4) {
                                const float4 f = f4[c4];
                                v[4 * c4 + 0] = __float_as_uint(f.x * __uint_as_float(v[4 * c4 + 0]));
                                v[4 * c4 + 1] = __float_as_uint(f.y * __uint_as_float(v[4 * c4 + 1]));
                                v[4 * c4 + 2] = __float_as_uint(f.z * __uint_as_float(v[4 * c4 + 2]));
                                v[4 * c4 + 3] = __float_as_uint(f.w * __uint_as_float(v[4 * c4 + 3]));
                            }
                        }
                        pack_pairs<32>(v, pk);
    #pragma unroll
                        for (int c = 0; c < 4; ++c)
                            *reinterpret_cast<uint4*>(zs + swz128(d, 32 * hh + 8 * c)) =
                                make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                    }
                    fence_async_smem();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&bars[B_ZFULL + x]);
                        if (GATED) mbar_arrive(&bars[B_EMPTYF + r % NF]);  // done with the chunk's factors
                    }
                    DN_TS(wq == 0, r, 13 + 4 * x);
                    // S_x^T -> bf16 (and fp32 out after the last chunk); the chunk's first
                    // product (the only reader of the bf16 copy) is complete
                    if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL + x], r & 1, abort_flag))) break;
                    DN_TS(wq == 0, r, 14 + 4 * x);
                    tc_fence_after();
    #pragma unroll 1
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t v[64], pk[32];
                        tmem_ld64(tmem + lane_base + tm_s(x) + 64 * hh, v);
                        pack_pairs<64>(v, pk);
                        store_sbf(x, hh, pk);
                        if (r == nch - 1) {
    #pragma unroll
                            for (int c = 0; c < 64; ++c) x_out[(int64_t)(64 * hh + c) * D + d] = __uint_as_float(v[c]);
                        }
                    }
                    tmem_wait_st();  // the bf16 copy's tensor-memory stores
                    fence_async_smem();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars[B_SBF + x]);
                    DN_TS(wq == 0, r, 15 + 4 * x);
                    if (GATED && r + 1 < nch) {
                        // S_x^T <- lambda[1:C] S_x^T of the next chunk before that chunk's update
                        // accumulates into it, off the chain (the update waits for this warp's
                        // next Z^T arrival); the bf16 copy above stays unscaled
                        if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_FULLF + (r + 1) % NF], ((r + 1) / NF) & 1,
                                                               abort_flag)))
                            break;
                        const float lam_next = ffac(r + 1)[kChunk];
                        tc_fence_after();
    #pragma unroll 1
                        for (int hh = 0; hh < 2; ++hh) {
                            uint32_t v[64];
                            tmem_ld64(tmem + lane_base + tm_s(x) + 64 * hh, v);
    #pragma unroll
                            for (int c = 0; c < 64; ++c) v[c] = __float_as_uint(lam_next * __uint_as_float(v[c]));
                            tmem_st32(tmem + lane_base + tm_s(x) + 64 * hh, *reinterpret_cast<uint32_t(*)[32]>(v));
                            tmem_st32(tmem + lane_base + tm_s(x) + 64 * hh + 32,
                                      *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                        }
                        tc_fence_before();
                    }
                }
            }
        }
    };
    if (mode == kModeHP) roles(std::true_type{});
    else roles(std::false_type{});

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicExch(p.err, kErrTimeout);
}

}  // namespace tcs
}  // namespace dn
