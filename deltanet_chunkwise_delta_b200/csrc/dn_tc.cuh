// Tensor-core (tcgen05 / TMEM / TMA) boundary pass for bf16, d_k = d_v = 128:
// every run of chunks from its true start state, with the outputs.
//
// Same per-chunk algorithm as dn_chain.cuh ("Linear Attention, Visualized",
// DeltaNet, "Complete per-chunk algorithm"), evaluated in the transposed
// domain so that every tensor-core product has M = 128:
//   T   = (I + B L)^{-1} B,  P = (Q K^T) o M_c   (from the UT pre-pass, dn_prep.cuh)
//   W^T = K^T T^T,  U^T = V^T T^T
//   [Z^T | O^T] = [U^T | 0] + S^T [-W^T | Q^T]   (one product, N = 128; for odd
//                                                 chunks [O^T | Z^T] from [Q^T | -W^T])
//   S^T <- S^T + Z^T K,   O^T += Z^T P^T
// S^T (d_v lanes x d_k columns, fp32) lives in tensor memory for the whole run.
// Its bf16 copy, and that of Z^T, also live in tensor memory, where the
// products read them as their A operand: the state chain never goes through
// shared memory, which the products' B operands, the TMA loads and the
// epilogues share.  W is written (negated) as token rows next to the chunk's
// query rows in its q/k stage, so that one product forms Z^T and S^T Q^T.
//
// Warp roles (512 threads):
//   warps 0-7   chain epilogue: Z^T -> bf16, S^T -> bf16 (tensor memory to
//               tensor memory), final state
//   warps 8-11  chunk-parallel epilogue: W^T -> -W token rows in shared
//               memory; O -> global (TMA store); lane 0 of warp 8 copies each
//               chunk's P tile in
//   warp 12     issues the state-chain products and the output product that
//               reads the chain's operand, one thread; owns the tensor memory
//   warp 13     TMA loads of k (3-stage ring) and q (3-stage ring; Gated DeltaNet:
//               bulk copies of the pre-pass's Q<- tile, 2 stages), one thread
//   warp 14     issues the chunk-parallel products (U^T, W^T), one thread
//   warp 15     TMA loads of v and bulk copies of T (2-stage ring), one thread
// The tensor pipe runs products in issue order, and a waiting issuer thread
// pays about 150 cycles per barrier even when the phase is already complete.
// So the chain issuer waits only for what its products need, and the parallel
// issuer, having done its own waits ahead of time, issues only inside the
// chain's two epilogue gaps (signalled by GAP1 / GAP2), where its products
// overlap the epilogues instead of delaying the next chain product.  Every wait on an
// mbarrier is bounded; on time-out the CTA drains, frees its tensor memory
// and reports DN_ERR_TIMEOUT through the error flag.
#pragma once

#include "dn_common.cuh"
#include "dn_kda_prep.cuh"
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
//   ring Q: NQ stages of [-W d0-63 | Q d0-63 | -W d64-127 | Q d64-127] (-W rows
//           written by the epilogue, q by TMA; [-W; Q] is one K-major operand of
//           128 token rows).  For odd chunks -W and Q swap places, so that the
//           product's [Z^T | O^T] columns alternate around one U^T / Z^T block
//           between two O^T buffers.
//   ring K: 3 stages of [K d0-63 | K d64-127] (TMA)
//   ring B: 2 stages of [V d0-63 | V d64-127 | T]
//   2 P tiles (chunk r's in buffer r % 2); O staging (two 64-column boxes of token rows)
// A chunk's ring-Q and ring-K stages are released together, by one commit after its
// state update (B_EMPTY + r % 6; the producer waits for chunk r - 3 before loading k of
// chunk r and for chunk r - NQ before its q).
// Gated DeltaNet: ring Q holds Q<- = diag(lambda[1:l]) Q from the pre-pass and has two
// stages, ring B stages also hold T' = T diag(lambda[1:l]) (the W<- factor), and each P
// buffer is followed by the chunk's row factors (lambda[l+1:C] per row, lambda[1:C]).
// Kimi Delta Attention (KDA, built on the gated layout): ring B stages hold K<- (the W
// factor, with T) in place of T', ring K holds K-> (the state update's operand, 2 stages),
// both from the KDA pre-pass, and the factors after each P tile are lambda[1:C] per key
// channel.
constexpr int NB = 2, NE = 6;
constexpr int Q_STAGE = 32768, K_STAGE = 16384;
__host__ __device__ constexpr int a_w(int c) { return (c & 1) ? 8192 : 0; }  // -W rows of chunk c
__host__ __device__ constexpr int a_q(int c) { return (c & 1) ? 0 : 8192; }  // Q rows of chunk c
constexpr int B_T = 16384, B_T2 = 24576;
constexpr int NBAR = 42;
constexpr int B_KL = 24576;  // KDA: K<- in a ring-B stage (two 64-channel boxes)
template <bool GATED, bool KDA = false>
struct TcLay {
    static constexpr int NQ = GATED ? 2 : 3;
    static constexpr int NK = KDA ? 2 : 3;
    static constexpr int OFF_K = NQ * Q_STAGE;
    static constexpr int OFF_B = OFF_K + NK * K_STAGE;
    static constexpr int B_STAGE = KDA ? 40960 : (GATED ? 32768 : 24576);  // V, T (, T' | K<-)
    static constexpr int PB_STRIDE = GATED ? 9216 : 8192;  // P tile (+ row factors)
    static constexpr int OFF_PB = OFF_B + NB * B_STAGE;
    static constexpr int OFF_OB = OFF_PB + 2 * PB_STRIDE;  // O staging
    static constexpr int OFF_BAR = OFF_OB + 16384;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM_USED = OFF_MISC + 64;
    static constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
};
static_assert(TcLay<false>::SMEM_BYTES <= 232448 && TcLay<true>::SMEM_BYTES <= 232448 &&
                  TcLay<true, true>::SMEM_BYTES <= 232448,
              "shared memory budget");
constexpr int SMEM_BYTES = TcLay<false>::SMEM_BYTES;

// tensor-memory columns (512 allocated): S^T fp32, [O^T (odd chunks) | U^T/Z^T |
// O^T (even chunks)] (one product of N = 128 writes Z^T and the chunk's O^T), W^T,
// Z^T bf16 (64 tokens in 32 columns), Gated DeltaNet: Z^T diag(lambda[l+1:C]) bf16 (the
// state update's operand), S^T bf16 (128 d_k in 64 columns)
constexpr uint32_t TM_S = 0, TM_O1 = 128, TM_ZU = 192, TM_O0 = 256, TM_WT = 320, TM_ZBF = 384, TM_ZBF2 = 416,
                   TM_SBF = 448;
__device__ __forceinline__ uint32_t tm_o(int c) { return (c & 1) ? TM_O1 : TM_O0; }   // O^T of chunk c
__device__ __forceinline__ uint32_t tm_c1(int c) { return (c & 1) ? TM_O1 : TM_ZU; }  // first product's D

// Barriers of a ring or of a double buffer come one per slot; a waiter on slot
// s for chunk r waits for that slot's (r / slots)-th completion.  Barriers
// completed by epilogue warps take one arrival per warp, after __syncwarp():
// each lane has already fenced its own writes or tensor-memory accesses.
enum : int {
    B_FULLQ = 0,     // +3: q of a ring-Q stage landed
    B_FULLK = 3,     // +3: k of a ring-K stage landed
    B_FULLB = 6,     // +2: v, T landed
    B_EMPTYB = 8,    // +2: stage of ring B consumed
    B_WUFULL = 10,   // W^T of the chunk ready in tensor memory
    B_WTFREE = 11,   // W^T columns read out
    B_WFULL = 12,    // -W rows of the chunk written to its ring-Q stage
    B_C1 = 13,       // [Z^T | O^T] product complete (bf16 S^T read)
    B_ZFULL = 14,    // bf16 Z^T written
    B_ZFREE = 15,    // fp32 U^T / Z^T columns read out
    B_SFULL = 16,    // S^T updated
    B_SBF = 17,      // bf16 S^T written
    B_OFULL = 18,    // O^T complete
    B_OFREE = 29,    // +2: O^T buffer read out and zeroed
    B_PFULL = 20,    // +2: P tile of the chunk copied into its buffer
    B_GAP1 = 22,     // +2: chain issuer: chunk's first product issued (one per chunk parity)
    B_OSTAGED = 24,  // O tile of the chunk staged as token rows
    B_OBFREE = 25,   // O staging buffer released by the chunk's store
    B_GAP2 = 26,     // +2: chain issuer: chunk's S^T update issued (one per chunk parity)
    B_UFULL = 28,    // U^T of the chunk ready in tensor memory
    B_DRAIN = 31,    // +2: drain of the chain issuer's / the parallel issuer's products
    B_STALL = 33,    // never completed: the wait of a test stall (Params::stall_chunk)
    B_EMPTY = 34,    // +6: chunk r's ring-Q and ring-K stages consumed (slot r % 6)
};
static_assert(B_EMPTY + NE <= NBAR, "barrier count");

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

// N fp32 values -> N / 2 packed bf16 pairs (the tensor-memory A-operand layout).
template <int N>
__device__ __forceinline__ void pack_pairs(const uint32_t* v, uint32_t* out) {
#pragma unroll
    for (int c = 0; c < N / 2; ++c) out[c] = pack_bf16(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1]));
}

// A warp's 32 rows (tensor-memory lanes 32 q .. 32 q + 31, i.e. d = 32 q + i) x
// 64 columns (tokens), read as 16-lane fragments: lo[g] from lanes 32 q .. + 15,
// hi[g] from lanes 32 q + 16 .. + 31, columns 8 g .. 8 g + 7.  Waits for the loads.
struct RowFrags {
    uint32_t lo[8][4], hi[8][4];
};
__device__ __forceinline__ void tmem_load_rows(uint32_t taddr_q, RowFrags& f) {
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        tmem_ld16x256(taddr_q + 8 * g, f.lo[g]);
        tmem_ld16x256(taddr_q + (16u << 16) + 8 * g, f.hi[g]);
    }
    tmem_wait_ld();
}
// The fragments of warp q, written transposed as bf16 token rows into two
// 64-column boxes of 128-byte swizzled rows (box d / 64 at box0 + (d / 64) *
// box_stride, column d % 64), scaled by `scale`: transposing matrix stores, 16
// bytes per token-row segment.
__device__ __forceinline__ void store_token_rows(const RowFrags& f, int q, uint8_t* box0, uint32_t box_stride,
                                                 float scale) {
    const int lane = threadIdx.x & 31;
    const uint32_t obox = saddr(box0) + (uint32_t)(q >> 1) * box_stride;
    const int dcol = 32 * (q & 1) + 8 * (lane >> 3);
#pragma unroll
    for (int g = 0; g < 8; ++g)
        stmatrix_x4_trans(obox + swz128(8 * g + (lane & 7), dcol),
                          pack_bf16(scale * __uint_as_float(f.lo[g][0]), scale * __uint_as_float(f.lo[g][1])),
                          pack_bf16(scale * __uint_as_float(f.lo[g][2]), scale * __uint_as_float(f.lo[g][3])),
                          pack_bf16(scale * __uint_as_float(f.hi[g][0]), scale * __uint_as_float(f.hi[g][1])),
                          pack_bf16(scale * __uint_as_float(f.hi[g][2]), scale * __uint_as_float(f.hi[g][3])));
}

// As store_token_rows (scale 1), with token row 8 g + (lane & 7) written to staging row
// prow[g] of this lane.
__device__ __forceinline__ void store_token_rows_mapped(const RowFrags& f, int q, uint8_t* box0, uint32_t box_stride,
                                                        const int (&prow)[8]) {
    const int lane = threadIdx.x & 31;
    const uint32_t obox = saddr(box0) + (uint32_t)(q >> 1) * box_stride;
    const int dcol = 32 * (q & 1) + 8 * (lane >> 3);
#pragma unroll
    for (int g = 0; g < 8; ++g)
        stmatrix_x4_trans(obox + swz128(prow[g], dcol), pack_bf16(__uint_as_float(f.lo[g][0]), __uint_as_float(f.lo[g][1])),
                          pack_bf16(__uint_as_float(f.lo[g][2]), __uint_as_float(f.lo[g][3])),
                          pack_bf16(__uint_as_float(f.hi[g][0]), __uint_as_float(f.hi[g][1])),
                          pack_bf16(__uint_as_float(f.hi[g][2]), __uint_as_float(f.hi[g][3])));
}

// toc: Gated Delta Product with n_h dividing 64, a map over out with boxes of 64 / n_h
// token rows (a chunk's outputs); otherwise the same as to.
// MULTI: the Gated Delta Product's instance (several steps per token); the others are
// compiled with one step per token.  KDA: Kimi Delta Attention's instance (with GATED).
template <bool GATED, bool MULTI = false, bool KDA = false>
static __global__ void __launch_bounds__(kThreadsTc, 1)
    k_tc_chain(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
               const __grid_constant__ CUtensorMap toc, Params p) {
    static_assert(!KDA || (GATED && !MULTI), "KDA runs on the gated layout, one step per token");
    using L = TcLay<GATED, KDA>;
    constexpr int NK = L::NK;
    constexpr int kUnit = KDA ? kKdaUnitBytes : unit_bytes(GATED);
    constexpr int kUnitQ = KDA ? kKdaUnitQL : kUnitQL;
    constexpr int kUnitFac = KDA ? kKdaUnitF : kUnitF;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int n_items = count_C(p.sched);
    if ((int)blockIdx.x >= n_items) return;
    const Item it = item_C(p.sched, blockIdx.x);

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    WaitCtl* ctl = reinterpret_cast<WaitCtl*>(smem + L::OFF_MISC + 8);
    volatile int* abort_flag = &ctl->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < L::NQ; ++s) mbar_init(&bars[B_FULLQ + s], 1);
        for (int s = 0; s < NK; ++s) mbar_init(&bars[B_FULLK + s], 1);
        for (int s = 0; s < NE; ++s) mbar_init(&bars[B_EMPTY + s], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[B_FULLB + s], 1);
            mbar_init(&bars[B_EMPTYB + s], 1);
            mbar_init(&bars[B_GAP1 + s], 1);
            mbar_init(&bars[B_GAP2 + s], 1);
            mbar_init(&bars[B_PFULL + s], 1);
        }
        mbar_init(&bars[B_UFULL], 1);
        mbar_init(&bars[B_WUFULL], 1);
        mbar_init(&bars[B_WTFREE], 4);
        mbar_init(&bars[B_WFULL], 4);
        mbar_init(&bars[B_C1], 1);
        mbar_init(&bars[B_ZFULL], 8);
        mbar_init(&bars[B_ZFREE], 8);
        mbar_init(&bars[B_SFULL], 1);
        mbar_init(&bars[B_SBF], 8);
        mbar_init(&bars[B_OFULL], 1);
        mbar_init(&bars[B_OFREE], 4);
        mbar_init(&bars[B_OFREE + 1], 4);
        mbar_init(&bars[B_OSTAGED], 4);
        mbar_init(&bars[B_OBFREE], 4);
        mbar_init(&bars[B_DRAIN], 1);
        mbar_init(&bars[B_DRAIN + 1], 1);
        mbar_init(&bars[B_STALL], 1);
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

    // start state and destination of the run
    const float* s0 = p.s0 ? p.s0 + it.seq * p.s0_sn + it.head * p.s0_sh : nullptr;
    const float* x_in = it.g == 0 ? s0 : p.wsS + (int64_t)(it.slot + it.g - 1) * D * D;
    // the last run writes the final state; with e_in_c, run 0 of a split chain writes its
    // end state where the segment scan reads it
    float* x_out = (it.g == it.G - 1 && p.sT) ? p.sT + it.seq * p.sT_sn + it.head * p.sT_sh : nullptr;
    if (it.g == 0 && it.G >= 2 && !p.sched.list && p.sched.e_in_c) x_out = p.wsH + (int64_t)it.slot * D * D;

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ rings K and Q
        // k of chunk r before its q: W^T(r) reads K a chunk before the first product
        // reads Q
        if (lane == 0 && nch > 0) {
            int issued_k = 0, issued_q = 0;
            for (int r = 0; r < nch; ++r) {
                const int t0 = it.tok0 + r * kChunk;
                const int sk = r % NK;
                if (r >= NK && !mbar_wait(&bars[B_EMPTY + (r - NK) % NE], ((r - NK) / NE) & 1, abort_flag)) break;
                mbar_expect_tx(&bars[B_FULLK + sk], 16384u);
                uint8_t* stk = smem + L::OFF_K + sk * K_STAGE;
                if constexpr (KDA) {
                    // K-> of the chunk, from the KDA pre-pass (two 8 KB boxes)
                    const uint8_t* kr =
                        p.wsT + ((size_t)(it.cbase + r) * p.sched.H + it.head) * kUnit + kKdaUnitKR;
#pragma unroll
                    for (int a = 0; a < 2; ++a) bulk_load(stk + a * 8192, kr + a * 8192, 8192, &bars[B_FULLK + sk]);
                } else {
#pragma unroll
                    for (int a = 0; a < 2; ++a)
                        tma_load_4d(stk + a * 8192, &tk, &bars[B_FULLK + sk], a * 64, it.head, t0, it.b);
                }
                issued_k = r + 1;
                const int sq = r % L::NQ;
                if (L::NQ < NK && r >= L::NQ &&
                    !mbar_wait(&bars[B_EMPTY + (r - L::NQ) % NE], ((r - L::NQ) / NE) & 1, abort_flag))
                    break;
                mbar_expect_tx(&bars[B_FULLQ + sq], 16384u);
                uint8_t* stq = smem + sq * Q_STAGE;
                if constexpr (GATED) {
                    // Q<- of the chunk, from the pre-pass (two 8 KB boxes)
                    const uint8_t* ql = p.wsT + ((size_t)(it.cbase + r) * p.sched.H + it.head) * kUnit + kUnitQ;
#pragma unroll
                    for (int a = 0; a < 2; ++a) bulk_load(stq + a_q(r) + a * 16384, ql + a * 8192, 8192, &bars[B_FULLQ + sq]);
                } else {
#pragma unroll
                    for (int a = 0; a < 2; ++a)
                        tma_load_4d(stq + a_q(r) + a * 16384, &tq, &bars[B_FULLQ + sq], a * 64, it.head, t0, it.b);
                }
                issued_q = r + 1;
                DN_TR(true, r, 24);
            }
            // the last loads issued must have landed before the CTA may exit (even after an abort)
            volatile int drain = 0;
            for (int r = issued_k - NK < 0 ? 0 : issued_k - NK; r < issued_k; ++r)
                mbar_wait(&bars[B_FULLK + (r % NK)], (r / NK) & 1, &drain, kDrainWaitNs);
            for (int r = issued_q - L::NQ < 0 ? 0 : issued_q - L::NQ; r < issued_q; ++r)
                mbar_wait(&bars[B_FULLQ + (r % L::NQ)], (r / L::NQ) & 1, &drain, kDrainWaitNs);
        }
    } else if (warp == kTmaBWarp) {
        // ------------------------------------------------------------ ring B: v, T
        if (lane == 0 && nch > 0) {
            const uint32_t bytes = 16384u + 8192u + (KDA ? 16384u : (GATED ? 8192u : 0u));
            int issued = 0;
            for (int r = 0; r < nch; ++r) {
                const int s = r & 1;
                if (r >= 2 && !mbar_wait(&bars[B_EMPTYB + s], ((r >> 1) - 1) & 1, abort_flag)) break;
                mbar_expect_tx(&bars[B_FULLB + s], bytes);
                uint8_t* st = smem + L::OFF_B + s * L::B_STAGE;
                const int t0 = it.tok0 + r * kChunk;
#pragma unroll
                for (int a = 0; a < 2; ++a)
                    tma_load_4d(st + a * 8192, &tv, &bars[B_FULLB + s], a * 64, it.head, t0, it.b);
                const uint8_t* unit = p.wsT + ((size_t)(it.cbase + r) * p.sched.H + it.head) * kUnit;
                bulk_load(st + B_T, unit, 8192, &bars[B_FULLB + s]);
                if constexpr (KDA) {
                    bulk_load(st + B_KL, unit + kKdaUnitKL, 8192, &bars[B_FULLB + s]);
                    bulk_load(st + B_KL + 8192, unit + kKdaUnitKL + 8192, 8192, &bars[B_FULLB + s]);
                } else if constexpr (GATED) {
                    bulk_load(st + B_T2, unit + kUnitT2, 8192, &bars[B_FULLB + s]);
                }
                issued = r + 1;
            }
            volatile int drain = 0;
            for (int r = issued - 2 < 0 ? 0 : issued - 2; r < issued; ++r)
                mbar_wait(&bars[B_FULLB + (r & 1)], (r >> 1) & 1, &drain, kDrainWaitNs);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ state-chain products
        // Per chunk: [Z^T | O^T] = [U^T | 0] + S^T [-W^T | Q^T] (one product of N = 128),
        // S^T += Z^T K, O^T += Z^T P^T.  After the first it opens a gap for the
        // chunk-parallel issuer.
        if (lane == 0 && nch > 0) {
            const uint32_t sb = saddr(smem);
            const uint32_t i_c1 = idesc_bf16(128, 128, false, false);
            const uint32_t i_c3 = idesc_bf16(128, 128, false, true);
            const uint32_t i_o = idesc_bf16(128, 64, false, false);
            const uint64_t dWQ = sdesc(sb, 16, 1024);           // [-W; Q] / [Q; -W] token rows, K-major
            const uint64_t dK = sdesc(sb + L::OFF_K, 8192, 1024);  // K, MN-major
            // the state update's A operand: Z^T, or for Gated DeltaNet Z^T diag(lambda[l+1:C])
            // (so that the update adds K->^T Z)
            constexpr uint32_t tm_zs = GATED && !KDA ? TM_ZBF2 : TM_ZBF;  // KDA: K-> in ring K
            const uint64_t dP = sdesc(sb + L::OFF_PB, 16, 1024);   // P^T, K-major (+ 8 KB for odd chunks)
            for (int r = 0; r < nch; ++r) {
                const int s = r & 1;
                const uint64_t stq = (uint64_t)(((r % L::NQ) * Q_STAGE) >> 4);
                const uint64_t stk = (uint64_t)(((r % NK) * K_STAGE) >> 4);
                DN_TR(true, r, 0);
                if (r + 1 == p.stall_chunk && !mbar_wait(&bars[B_STALL], 0, abort_flag)) break;
                const bool ready = mbar_wait4(&bars[B_WFULL], r & 1, &bars[B_SBF], r & 1, &bars[B_UFULL], r & 1,
                                              &bars[B_OFREE + s], (r >> 1) & 1, abort_flag);
                if (!ready) break;
                DN_TR(true, r, 3);
                tc_fence_after();
                // [Z^T | O^T] = [U^T | 0] + S^T [-W^T | Q^T]  (odd chunks: [O^T | Z^T])
                const uint32_t d1 = tm_c1(r);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint64_t o = (uint64_t)(((j >> 2) * 16384 + (j & 3) * 32) >> 4);
                    umma_bf16_ts(tmem + d1, tmem + TM_SBF + 8 * j, dWQ + stq + o, i_c1, 1u);
                }
                umma_commit(&bars[B_C1]);
                mbar_arrive(&bars[B_GAP1 + s]);
                DN_TR(true, r, 1);
                if (!(KDA ? mbar_wait2(&bars[B_ZFULL], r & 1, &bars[B_FULLK + r % NK], (r / NK) & 1, abort_flag)
                          : mbar_wait(&bars[B_ZFULL], r & 1, abort_flag)))
                    break;
                DN_TR(true, r, 10);
                tc_fence_after();
                // S^T += Z^T K
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    umma_bf16_ts(tmem + TM_S, tmem + tm_zs + 8 * j, dK + stk + (uint64_t)((j * 2048) >> 4), i_c3,
                                 1u);
                umma_commit(&bars[B_SFULL]);
                // the chunk's -W, q and k are read by the products above (and k by W^T of
                // the chunk, complete before its -W rows were written)
                umma_commit(&bars[B_EMPTY + r % NE]);
                mbar_arrive(&bars[B_GAP2 + s]);
                {
                    // O^T += Z^T P^T
                    if (!mbar_wait(&bars[B_PFULL + s], (r >> 1) & 1, abort_flag)) break;
                    tc_fence_after();
                    const uint64_t pofs = (uint64_t)((s * L::PB_STRIDE) >> 4);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_bf16_ts(tmem + tm_o(r), tmem + TM_ZBF + 8 * j, dP + pofs + (uint64_t)((j * 32) >> 4),
                                     i_o, 1u);
                    umma_commit(&bars[B_OFULL]);
                }
                DN_TR(true, r, 11);
            }
            umma_drain(&bars[B_DRAIN]);
        }
    } else if (warp == kParMmaWarp) {
        // ------------------------------------------------------------ chunk-parallel products
        // W^T and U^T of chunk r+1, issued in the chain's gaps so that they never
        // queue in front of a chain product: W^T after chunk r's first product is
        // issued (its -W rows are converted while the chain runs), U^T after chunk
        // r's S^T update is issued (Z^T(r) has been read out of the columns U^T
        // overwrites by then).  Other waits come before each gap.
        if (lane == 0 && nch > 0) {
            const uint32_t sb = saddr(smem);
            const uint32_t i_tt = idesc_bf16(128, 64, true, false);
            const uint64_t dKT = sdesc(sb + L::OFF_K, 8192, 1024);     // K^T, MN-major
            const uint64_t dVT = sdesc(sb + L::OFF_B, 8192, 1024);        // V^T, MN-major
            const uint64_t dT = sdesc(sb + L::OFF_B + B_T, 16, 1024);     // T^T, K-major
            // W = T K, or for Gated DeltaNet W<- = T' K with T' = T diag(lambda[1:l])
            const uint64_t dTw = GATED && !KDA ? sdesc(sb + L::OFF_B + B_T2, 16, 1024) : dT;
            // KDA: W = T K<- with K<- in ring B
            const uint64_t dKLT = sdesc(sb + L::OFF_B + B_KL, 8192, 1024);
            auto issue_w = [&](int c) {
                const uint64_t stk = KDA ? (uint64_t)(((c & 1) * L::B_STAGE) >> 4)
                                         : (uint64_t)(((c % NK) * K_STAGE) >> 4);
                const uint64_t stb = (uint64_t)(((c & 1) * L::B_STAGE) >> 4);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    umma_bf16(tmem + TM_WT, (KDA ? dKLT : dKT) + stk + (uint64_t)((j * 2048) >> 4),
                              dTw + stb + (uint64_t)((j * 32) >> 4), i_tt, j > 0);
                umma_commit(&bars[B_WUFULL]);
            };
            // U^T of chunk c; its ring-B stage is consumed after it (W^T came first)
            auto issue_u = [&](int c) {
                const int s = c & 1;
                const uint64_t stb = (uint64_t)((s * L::B_STAGE) >> 4);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    umma_bf16(tmem + TM_ZU, dVT + stb + (uint64_t)((j * 2048) >> 4),
                              dT + stb + (uint64_t)((j * 32) >> 4), i_tt, j > 0);
                umma_commit(&bars[B_UFULL]);
                umma_commit(&bars[B_EMPTYB + s]);
            };
            // (KDA: W^T reads K<- from ring B; ring K's K-> is the state update's alone)
            auto wait_data = [&](int c) -> bool {
                if constexpr (KDA) return mbar_wait(&bars[B_FULLB + (c & 1)], (c >> 1) & 1, abort_flag);
                return mbar_wait2(&bars[B_FULLK + c % NK], (c / NK) & 1, &bars[B_FULLB + (c & 1)], (c >> 1) & 1,
                                  abort_flag);
            };
            bool ok = wait_data(0);
            if (ok) {
                tc_fence_after();
                issue_w(0);
                issue_u(0);
            }
            for (int r = 0; ok && r + 1 < nch; ++r) {
                // gap 1: chunk r + 1's data, chunk r's W^T read out
                if (!wait_data(r + 1) || !mbar_wait(&bars[B_WTFREE], r & 1, abort_flag) ||
                    !mbar_wait(&bars[B_GAP1 + (r & 1)], (r >> 1) & 1, abort_flag))
                    break;
                DN_TR(true, r, 6);
                tc_fence_after();
                issue_w(r + 1);
                DN_TR(true, r, 7);
                // gap 2: Z^T(r) read out of the U^T / Z^T columns (before its S^T update)
                if (!mbar_wait(&bars[B_ZFREE], r & 1, abort_flag) ||
                    !mbar_wait(&bars[B_GAP2 + (r & 1)], (r >> 1) & 1, abort_flag))
                    break;
                tc_fence_after();
                issue_u(r + 1);
                DN_TR(true, r, 4);
            }
            umma_drain(&bars[B_DRAIN + 1]);
        }
    } else if (warp >= 8 && warp < 12) {
        // ------------------------------------------------------------ chunk-parallel epilogue
        const int q = warp - 8;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        int p_issued = 0;
        // P tile of chunk c into buffer c % 2 (one thread); Gated DeltaNet: followed by the
        // chunk's row factors
        auto issue_p = [&](int c) {
            ++p_issued;
            const uint8_t* unit = p.wsT + ((size_t)(it.cbase + c) * p.sched.H + it.head) * kUnit;
            uint8_t* buf = smem + L::OFF_PB + (c & 1) * L::PB_STRIDE;
            mbar_expect_tx(&bars[B_PFULL + (c & 1)], 8192u + (GATED ? (uint32_t)kUnitFBytes : 0u));
            static_assert(kKdaUnitFBytes == kUnitFBytes, "row factors of one size");
            bulk_load(buf, unit + 8192, 8192, &bars[B_PFULL + (c & 1)]);
            if constexpr (GATED) bulk_load(buf + 8192, unit + kUnitFac, kUnitFBytes, &bars[B_PFULL + (c & 1)]);
        };
        // O^T of chunk c -> out: read out of tensor memory (and zeroed for the next
        // chunk's first product, which accumulates into it), staged as token rows (the
        // TMA box layout of out) and written by one TMA store per box; a chunk that
        // ends inside the run's last 64 tokens is written with bounded 16-byte stores.
        // Gated Delta Product: rows are steps, and only a token's last step is written,
        // to its token row (bounded stores).
        __nv_bfloat16* og = static_cast<__nv_bfloat16*>(p.o) + it.b * p.o_sb + it.head * p.o_sh;
        const int nh = MULTI && p.nh > 1 ? p.nh : 1;  // steps per token (Gated Delta Product)
        // Gated Delta Product with n_h dividing 64: a full chunk's outputs (a token's last
        // step) are packed into staging rows 0 .. 64 / n_h - 1 and written with one TMA store
        // per box; the other steps' rows go to distinct rows past them
        const bool packed_o = MULTI && nh > 1 && kChunk % nh == 0;
        int prow[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            const int t = 8 * g + (lane & 7), kept = kChunk / nh;
            prow[g] = !MULTI ? t : (t + 1) % nh == 0 ? t / nh : kept + t % (kChunk - kept);
        }
        uint8_t* ob = smem + L::OFF_OB;
        auto store_o = [&](int c) -> bool {
            // read out and zero the columns first: the next chunk's first product waits
            // for them
            tc_fence_after();
            RowFrags f;
            tmem_load_rows(tmem + lane_base + tm_o(c), f);
            tmem_zero32(tmem + lane_base + tm_o(c));
            tmem_zero32(tmem + lane_base + tm_o(c) + 32);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_OFREE + (c & 1)]);
            DN_TR(q == 0, c, 21);
            // the staging buffer is released by chunk c - 1's store
            if (c >= 1 && !__all_sync(0xffffffffu, mbar_wait(&bars[B_OBFREE], (c - 1) & 1, abort_flag)))
                return false;
            const int t0 = it.tok0 + c * kChunk;
            const bool full = t0 + kChunk <= it.tok1;
            if (MULTI && packed_o && full) store_token_rows_mapped(f, q, ob, 8192, prow);
            else store_token_rows(f, q, ob, 8192, 1.f);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_OSTAGED]);
            DN_TR(q == 0, c, 28);
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_OSTAGED], c & 1, abort_flag))) return false;
            if (full && (nh == 1 || packed_o)) {
                if (q == 0 && lane == 0) {
                    const CUtensorMap* om = MULTI && nh > 1 ? &toc : &to;
                    const int r0 = MULTI && nh > 1 ? t0 / nh : t0;
                    tma_store_4d(om, ob, 0, it.head, r0, it.b);
                    tma_store_4d(om, ob + 8192, 64, it.head, r0, it.b);
                    bulk_commit();
                    bulk_wait_read0();
                }
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int id = 32 * q + lane + 128 * k, t = id >> 4, dc = id & 15;
                    const uint4 row = *reinterpret_cast<const uint4*>(ob + (dc >> 3) * 8192 + swz128(t, (dc & 7) * 8));
                    const int m = t0 + t;
                    if (m < it.tok1 && (m + 1) % nh == 0)
                        *reinterpret_cast<uint4*>(og + (int64_t)(m / nh) * p.o_st + 8 * dc) = row;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_OBFREE]);
            DN_TR(q == 0, c, 26);
            return true;
        };
        {
            // both O^T buffers start at zero: the first product accumulates into them
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                tmem_zero32(tmem + lane_base + tm_o(b));
                tmem_zero32(tmem + lane_base + tm_o(b) + 32);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_OFREE]);
                mbar_arrive(&bars[B_OFREE + 1]);
            }
        }
        for (int r = 0; r < nch; ++r) {
            uint8_t* stage = smem + (r % L::NQ) * Q_STAGE;
            // W^T (tensor memory, d_k lanes) -> -W token rows in the chunk's ring-Q stage,
            // once the stage holds the chunk (its previous chunk's products are done)
            if (!__all_sync(0xffffffffu, mbar_wait2(&bars[B_WUFULL], r & 1, &bars[B_FULLQ + r % L::NQ],
                                                    (r / L::NQ) & 1, abort_flag)))
                break;
            DN_TR(q == 0, r, 13);
            tc_fence_after();
            {
                RowFrags f;
                tmem_load_rows(tmem + lane_base + TM_WT, f);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_WTFREE]);
                store_token_rows(f, q, stage + a_w(r), 16384, -1.f);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_WFULL]);
            DN_TR(q == 0, r, 14);
            if (r >= 1) {
                // chunk r - 1 complete: copy in chunk r + 1's P tile (into chunk r - 1's
                // buffer), write out O of chunk r - 1
                if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_OFULL], (r - 1) & 1, abort_flag))) break;
                if (q == 0 && lane == 0 && r + 1 < nch) issue_p(r + 1);
                if (!store_o(r - 1)) break;
            } else if (q == 0 && lane == 0) {
                issue_p(0);
                if (nch > 1) issue_p(1);
            }
        }
        if (nch > 0 && !*abort_flag &&
            __all_sync(0xffffffffu, mbar_wait(&bars[B_OFULL], (nch - 1) & 1, abort_flag)))
            store_o(nch - 1);
        // the last P copies must have landed, and the TMA stores of O completed,
        // before the CTA may exit (even after an abort); P copies go to chunks 0, 1, ...
        // in order, so copy c completes phase c / 2 of buffer c % 2
        if (lane == 0) {
            volatile int drain = 0;
            for (int c = p_issued - 2 < 0 ? 0 : p_issued - 2; c < p_issued; ++c)
                mbar_wait(&bars[B_PFULL + (c & 1)], (c >> 1) & 1, &drain, kDrainWaitNs);
        }
        if (q == 0 && lane == 0) bulk_wait0();
    } else if (warp < 8) {
        // ------------------------------------------------------------ chain epilogue
        // Warp w handles d_v rows 32 (w % 4) .. + 31 (its tensor-memory lane quarter)
        // and half h = w / 4 of the columns.
        const int wq = warp & 3, h = warp >> 2;
        const int d = 32 * wq + lane;  // d_v row of S^T, Z^T
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        // the state entering chunk c of the run (for a backward pass): row = global chunk
        // index; this thread's column d of key rows 64 h .. + 63 (a warp writes 128
        // contiguous bytes of each row)
        // Gated DeltaNet: the row factors of chunk c (lambda[l+1:C] for rows l = 0..63, then
        // lambda[1:C]), in its P buffer from B_PFULL until the chunk's output product is
        // complete
        auto pfac = [&](int c) {
            return reinterpret_cast<const float*>(smem + L::OFF_PB + (c & 1) * L::PB_STRIDE + 8192);
        };
        // Gated DeltaNet: this thread's 64 values of S^T times lambda[1:C] (f[64]), in
        // registers.  KDA: its columns (key channels 64 h .. 64 h + 63) of S^T in tensor memory
        // times lambda[1:C] of their channel, 32 columns at a time (the caller has written them)
        auto rescale_state = [&](uint32_t(&v)[64], const float* f) {
            const float lam = f[kChunk];
#pragma unroll
            for (int c = 0; c < 64; ++c) v[c] = __float_as_uint(lam * __uint_as_float(v[c]));
        };
        auto rescale_state_tm = [&](const float* f) {
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t w[32];
                const uint32_t ta = tmem + lane_base + TM_S + 64 * h + 32 * hf;
                tmem_ld32(ta, w);
                const float* fh = f + 64 * h + 32 * hf;
#pragma unroll
                for (int c = 0; c < 32; ++c) w[c] = __float_as_uint(fh[c] * __uint_as_float(w[c]));
                tmem_st32(ta, w);
            }
        };
        auto store_chunk_state = [&](int c, const uint32_t(&v)[64]) {
            const int64_t row = (int64_t)it.cbase + c;
            if (!p.cs || row >= p.cs_rows) return;
            float* dst = p.cs + row * p.cs_sc + it.head * p.cs_sh + d;
#pragma unroll
            for (int cc = 0; cc < 64; ++cc) dst[(int64_t)(64 * h + cc) * D] = __uint_as_float(v[cc]);
        };
        bool live = true;
        {
            uint32_t v[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const int a = 64 * h + c;
                float x = 0.f;
                if (x_in) x = x_in[(int64_t)a * D + d];
                v[c] = __float_as_uint(x);
            }
            if (nch == 0) {
                if (x_out)
                    for (int c = 0; c < 64; ++c) x_out[(int64_t)(64 * h + c) * D + d] = __uint_as_float(v[c]);
            } else {
                store_chunk_state(0, v);
                uint32_t pk[32];
                pack_pairs<64>(v, pk);
                tmem_st32(tmem + lane_base + TM_SBF + 32 * h, pk);
                if constexpr (GATED) {
                    // Gated DeltaNet: the update of chunk 0 adds K->^T Z to lambda[1:C] S (the
                    // chunk's factors arrive with its P tile); KDA: Diag(lambda[1:C]) S, this
                    // thread's key channels 64 h .. 64 h + 63
                    live = __all_sync(0xffffffffu, mbar_wait(&bars[B_PFULL], 0, abort_flag));
                    if (!KDA && live) rescale_state(v, pfac(0));
                }
                tmem_st32(tmem + lane_base + TM_S + 64 * h, *reinterpret_cast<uint32_t(*)[32]>(v));
                tmem_st32(tmem + lane_base + TM_S + 64 * h + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                if (KDA && live) rescale_state_tm(pfac(0));
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && live) mbar_arrive(&bars[B_SBF]);
        for (int r = 0; live && r < nch; ++r) {
            // Z^T -> bf16 (A operand of the S^T update and of O^T += Z^T P^T), once the
            // previous chunk's O^T += Z^T P^T has read the previous one
            DN_TR(warp == 0, r, 27);
            if (r >= 1 &&
                !__all_sync(0xffffffffu, mbar_wait(&bars[B_OFULL], (r - 1) & 1, abort_flag)))
                break;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_C1], r & 1, abort_flag))) break;
            DN_TR(warp == 0, r, 16);
            tc_fence_after();
            {
                uint32_t v[32], pk[16];
                tmem_ld32(tmem + lane_base + TM_ZU + 32 * h, v);
                pack_pairs<32>(v, pk);
                tmem_st16(tmem + lane_base + TM_ZBF + 16 * h, pk);
                if constexpr (GATED && !KDA) {
                    // Z^T diag(lambda[l+1:C]) for the state update (this half's 32 tokens)
                    const float4* f4 = reinterpret_cast<const float4*>(pfac(r) + 32 * h);
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 f = f4[c4];
                        v[4 * c4 + 0] = __float_as_uint(f.x * __uint_as_float(v[4 * c4 + 0]));
                        v[4 * c4 + 1] = __float_as_uint(f.y * __uint_as_float(v[4 * c4 + 1]));
                        v[4 * c4 + 2] = __float_as_uint(f.z * __uint_as_float(v[4 * c4 + 2]));
                        v[4 * c4 + 3] = __float_as_uint(f.w * __uint_as_float(v[4 * c4 + 3]));
                    }
                    pack_pairs<32>(v, pk);
                    tmem_st16(tmem + lane_base + TM_ZBF2 + 16 * h, pk);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_ZFULL]);
                mbar_arrive(&bars[B_ZFREE]);
            }
            DN_TR(warp == 0, r, 17);
            // S^T -> bf16 (and fp32 out after the last chunk); the chunk's first product
            // (the only reader of the bf16 copy) is complete
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
                if (r + 1 < nch) store_chunk_state(r + 1, v);
                if (GATED && r + 1 < nch) {
                    // S^T <- lambda[1:C] S^T of the next chunk before that chunk's update
                    // accumulates into it (complete before this warp's next Z^T arrival, which
                    // the update waits for); the bf16 copy above stays unscaled
                    if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_PFULL + ((r + 1) & 1)], ((r + 1) >> 1) & 1,
                                                           abort_flag)))
                        break;
                    if constexpr (KDA) {
                        rescale_state_tm(pfac(r + 1));
                    } else {
                        rescale_state(v, pfac(r + 1));
                        tmem_st32(tmem + lane_base + TM_S + 64 * h, *reinterpret_cast<uint32_t(*)[32]>(v));
                        tmem_st32(tmem + lane_base + TM_S + 64 * h + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                    }
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
