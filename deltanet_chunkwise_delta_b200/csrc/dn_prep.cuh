// UT pre-pass: the chunk-local factors of every (chunk, head), computed once.
//
// "Context Parallelism for DeltaNet", section 2, step 1: the WY factors of a
// chunk depend only on that chunk's keys and step sizes, so every chunk can be
// processed in parallel.  Per (chunk r, head) this kernel forms
//   G_r = [Q_r; K_r] K_r^T                 (one tcgen05 product, M = 128)
//   L_r = (K_r K_r^T) o M_c^-,    T_r = (I + B_r L_r)^{-1} B_r
//   P_r = (Q_r K_r^T) o M_c               (inclusive causal mask)
// ("Linear Attention, Visualized", DeltaNet, "Complete per-chunk algorithm")
// and stores T_r and P_r as two bf16 64 x 64 tiles (16 KB per unit, T first)
// whose rows are 128 bytes with the 128-byte swizzle: exactly the
// shared-memory layout in which the chain kernel uses T^T and P^T as
// tensor-core operands (it copies each tile in with one bulk copy).  Both tiles
// are built in shared memory (in scratch space that is free at that point of
// the unit) and written out with one bulk copy each.
// W_r = T_r K_r and U_r = T_r V_r are formed later, next to the state chain.
//
// The 64 x 64 solve is blocked in 16 x 16 blocks: N = (I + A)^{-1} with
// A = B L; each diagonal block by forward substitution (one warp per block,
// one column per lane, fp32), then N_ij = -N_ii sum_{k=j}^{i-1} A_ik N_kj in
// order of i - j with tf32 mma.sync, and T = N B.
// Gated DeltaNet ("Linear Attention, Visualized", section "Gated DeltaNet
// (GDN)", complete per-chunk algorithm): with the running sums c_l of the
// chunk's log decays, Gamma[l][i] = lambda[i+1:l] = exp(c_l - c_i) multiplies
// both halves of G (L = (K K^T o Gamma) o M_c^-, P = (Q K^T o Gamma) o M_c),
// and a third tile T' = T diag(lambda[1:l]) = T diag(exp(c_l)) gives
// W<- = T K<- = T' K to the chain kernels.  The unit also carries what the chain
// kernels would otherwise compute from the log decays next to the state chain: the
// decayed queries Q<- = diag(lambda[1:l]) Q (the unit's q boxes scaled per token
// row, in the layout the tensor cores read), and the row factors lambda[l+1:C] =
// exp(c_C - c_l) and lambda[1:C] = exp(c_C) (K-> = diag(lambda[l+1:C]) K enters the
// state update as diag(lambda[l+1:C]) Z, the state's decay as lambda[1:C]).
// Gated Delta Product (same page, "GDP as GDN over a virtual sequence"): a chunk is 64
// virtual steps m (write j of token t is m = n_h t + j; k, v and beta hold one row per
// step); the step's query is that of token m / n_h (read only on a token's last step, the
// others' outputs are not stored) and its log decay that of the token on its first step,
// 0 on the others.  The unit's q box is loaded from token (first step) / n_h and expanded
// to one row per step in shared memory before the Gram product.
// One CTA of 4 warps per (chunk, head) at a time, six CTAs per SM, so the latency of
// the solve is hidden by parallelism across chunks.  A CTA's shared memory is one 32 KB
// region that holds the unit's q/k tile until the product has read it, and then the
// solve's blocks, the P tile (staged where N is written later), the T tile (staged where
// A was) and, gated, the T' tile (staged in the next 8 KB once N is read); the next
// unit's tile is loaded as soon as the T tile is built, the boxes over the T (and T')
// staging once the copies have read it.
#pragma once

#include "dn_chain.cuh"
#include "dn_common.cuh"
#include "dn_sm100.cuh"
#include "dn_warp_gemm.cuh"

namespace dn {

#ifdef DN_TRACE
static __device__ unsigned long long g_dn_trace_prep[16 * 8];
#define DN_TRP(k, slot)                                                               \
    do {                                                                              \
        if (blockIdx.x == 0 && (k) < 16 && threadIdx.x == 0) {                         \
            unsigned long long t_;                                                    \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                    \
            g_dn_trace_prep[(k) * 8 + (slot)] = t_;                                   \
        }                                                                             \
    } while (0)
#else
#define DN_TRP(k, slot) \
    do {                \
    } while (0)
#endif

constexpr int kPrepThreads = 128;
template <bool GATED>
constexpr int prep_ctas_per_sm() { return 6; }
constexpr int kPrepCtasPerSm = prep_ctas_per_sm<false>();
constexpr int kBlkLd = 20;  // fp32 16 x 16 blocks, 16-byte aligned rows
constexpr int kBlkFloats = 16 * kBlkLd;

// Shared memory of the pre-pass (byte offsets from a 1024-aligned base).  The
// region [0, 32 KB) holds [Q d0-63 | K d0-63 | Q d64-127 | K d64-127] while the
// q/k tile is loaded and read by the product, then the blocks of the solve:
template <bool GATED>
struct PrepSmemT {
    static constexpr int OFF_QK = 0;
    static constexpr int OFF_A = 0;                               // 10 blocks of A = B L; later the T tile
    static constexpr int OFF_N = OFF_A + 10 * kBlkFloats * 4;     // 10 blocks of N; before them the P tile
    static constexpr int OFF_X = OFF_N + 10 * kBlkFloats * 4;     // 5 staging blocks of the off-diagonal solve
    static constexpr int OFF_T2 = 8192;                           // gated: the T' tile, once N is read
    static constexpr int OFF_BETA = 32768;                        // 2 x 64 step sizes
    static constexpr int OFF_G = OFF_BETA + 2 * kChunk * 4;       // gated: 2 x 64 log decays
    static constexpr int OFF_C = OFF_G + (GATED ? 2 * kChunk * 4 : 0);  // gated: 64 running sums
    static constexpr int OFF_LAM = OFF_C + (GATED ? kChunk * 4 : 0);    // gated: exp of those
    static constexpr int OFF_BAR = OFF_LAM + (GATED ? kChunk * 4 : 0);  // FULL, GDONE, DRAIN
    static constexpr int OFF_MISC = OFF_BAR + 24;                 // TMEM address, then the WaitCtl at + 8
    static constexpr int USED = OFF_MISC + 24;
    static constexpr int TOTAL = USED + 1024;                     // slack for 1024-byte alignment
};
using PrepSmem = PrepSmemT<false>;
static_assert(PrepSmem::OFF_X + 5 * kBlkFloats * 4 <= 32768, "solve blocks fit the q/k region");
static_assert(PrepSmem::OFF_N + 8192 <= PrepSmem::OFF_X, "P staging fits the N blocks");
static_assert((PrepSmemT<false>::TOTAL + 1024) * prep_ctas_per_sm<false>() <= 228 * 1024, "pre-pass shared memory");
static_assert((PrepSmemT<true>::TOTAL + 1024) * prep_ctas_per_sm<true>() <= 228 * 1024, "pre-pass shared memory");

__device__ __forceinline__ int blk_index(int bi, int bj) { return bi * (bi + 1) / 2 + bj; }

// bf16 pair * f, rounded to nearest-even.
__device__ __forceinline__ uint32_t scale_pair(uint32_t w, float f) {
    return sm100::pack_bf16(__uint_as_float(w << 16) * f, __uint_as_float(w & 0xffff0000u) * f);
}

// acc (16 x 16, two n8 tiles) += A (16 x 16) * B (16 x 16), tf32 inputs, fp32 accumulate.
__device__ __forceinline__ void mm16_tf32(float (&acc)[2][4], const float* A, const float* B) {
    blk16_tf32<kBlkLd>(acc, A, B);
}

__device__ __forceinline__ void st_blk(float* C, const float (&acc)[2][4], float scale) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        *reinterpret_cast<float2*>(C + g * kBlkLd + 8 * nt + 2 * t) =
            make_float2(scale * acc[nt][0], scale * acc[nt][1]);
        *reinterpret_cast<float2*>(C + (g + 8) * kBlkLd + 8 * nt + 2 * t) =
            make_float2(scale * acc[nt][2], scale * acc[nt][3]);
    }
}

// N_ij = -N_ii Y for a finished sum Y = sum_k A_ik N_kj held in acc (one warp).
__device__ __forceinline__ void finish_block(float* Nblk, float* X, int i, int j, const float (&acc)[2][4]) {
    st_blk(X, acc, 1.f);
    __syncwarp();
    float out[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    mm16_tf32(out, Nblk + blk_index(i, i) * kBlkFloats, X);
    st_blk(Nblk + blk_index(i, j) * kBlkFloats, out, -1.f);
}

__device__ __forceinline__ void ld_blk(float (&acc)[2][4], const float* C) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const float2 a = *reinterpret_cast<const float2*>(C + g * kBlkLd + 8 * nt + 2 * t);
        const float2 b = *reinterpret_cast<const float2*>(C + (g + 8) * kBlkLd + 8 * nt + 2 * t);
        acc[nt][0] = a.x; acc[nt][1] = a.y; acc[nt][2] = b.x; acc[nt][3] = b.y;
    }
}

// MULTI: the Gated Delta Product's instance (several steps per token); the others are
// compiled with one step per token.
template <bool GATED, bool MULTI = false>
static __global__ void __launch_bounds__(kPrepThreads, prep_ctas_per_sm<GATED>())
    k_ut_prep(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk, Params p) {
    using L = PrepSmemT<GATED>;
    constexpr int kUnit = unit_bytes(GATED);
    extern __shared__ uint8_t prep_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(prep_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float* Ablk = reinterpret_cast<float*>(smem + L::OFF_A);
    float* Nblk = reinterpret_cast<float*>(smem + L::OFF_N);
    float* Xs = reinterpret_cast<float*>(smem + L::OFF_X);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);  // [0] FULL, [1] GDONE, [2] DRAIN
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    sm100::WaitCtl* ctl = reinterpret_cast<sm100::WaitCtl*>(smem + L::OFF_MISC + 8);
    volatile int* abort_flag = &ctl->abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.sched.H;
    const int nh = MULTI && p.nh > 1 ? p.nh : 1;  // steps per token (Gated Delta Product)
    const int units = count_chunks(p.sched) * H;
    if ((int)blockIdx.x >= units) return;

    if (tid == 0) {
        sm100::mbar_init(&bars[0], 1);
        sm100::mbar_init(&bars[1], 1);
        sm100::mbar_init(&bars[2], 1);
        sm100::wait_ctl_init(ctl, p.wait_ns);
        sm100::mbar_fence_init();
    }
    if (warp == 0) {
        sm100::tmem_alloc(tmem_slot, 64);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // q/k tile of unit u (TMA, thread 0) and its step sizes into beta buffer `bb`
    // (cp.async, zero past the chunk's last token, which zeroes T's rows and
    // columns there; one group)
    // With t_staged, the T tile of the previous unit is being copied out of the first
    // 8 KB of the region (gated: and T' out of the next 8 KB): the other boxes go first,
    // the boxes that overwrite the staging once the copies have read it.
    auto issue = [&](int u, int bb, bool t_staged) {
        const int id = u / H, head = u % H;
        int b, t0, t1;
        chunk_range(p.sched, id, b, t0, t1);
        const int tq0 = nh > 1 ? t0 / nh : t0;  // token of the chunk's first step (q is per token)
        if (tid == 0) {
            sm100::mbar_expect_tx(&bars[0], 32768u);
            if (!GATED) sm100::tma_load_4d(smem + L::OFF_QK + 8192, &tk, &bars[0], 0, head, t0, b);
            sm100::tma_load_4d(smem + L::OFF_QK + 16384, &tq, &bars[0], 64, head, tq0, b);
            sm100::tma_load_4d(smem + L::OFF_QK + 16384 + 8192, &tk, &bars[0], 64, head, t0, b);
            if (t_staged) sm100::bulk_wait_read0();
            sm100::tma_load_4d(smem + L::OFF_QK, &tq, &bars[0], 0, head, tq0, b);
            if (GATED) sm100::tma_load_4d(smem + L::OFF_QK + 8192, &tk, &bars[0], 0, head, t0, b);
        }
        if (tid < kChunk) {
            const bool ok = tid < t1 - t0;
            const float* src = p.beta + b * p.b_sb + (int64_t)(t0 + (ok ? tid : 0)) * p.b_st + head * p.b_sh;
            cp_async4(smem_addr(smem + L::OFF_BETA + (bb * kChunk + tid) * 4), src, ok ? 4 : 0);
            if constexpr (GATED) {
                // log decays of the chunk (0 past its end: the pad rows are identity steps;
                // Gated Delta Product: the token's on its first step, 0 on the others)
                const int m = t0 + (ok ? tid : 0);
                const bool gok = ok && (nh == 1 || m % nh == 0);
                const float* gsrc = p.g + b * p.g_sb + (int64_t)(nh > 1 ? m / nh : m) * p.g_st + head * p.g_sh;
                cp_async4(smem_addr(smem + L::OFF_G + (bb * kChunk + tid) * 4), gsrc, gok ? 4 : 0);
            }
        }
        cp_async_commit();
    };

    const uint32_t i_g = sm100::idesc_bf16(128, 64, false, false);
    const uint64_t dQK = sm100::sdesc(sm100::saddr(smem + L::OFF_QK), 16, 1024);
    bool in_flight = true;
    issue(blockIdx.x, 0, false);
    int it_ = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++it_) {
        const int bb = it_ & 1;
        DN_TRP(it_, 0);
        const bool got = sm100::mbar_wait(&bars[0], it_ & 1, abort_flag);
        cp_async_wait<0>();
        if (__syncthreads_or(!got)) break;
        in_flight = false;
        DN_TRP(it_, 1);
        if (GATED && nh > 1) {
            // Gated Delta Product: step row m of the q boxes takes token row (t0 + m) / n_h - tq0
            // of the loaded boxes (128-byte rows whose 16-byte pieces are swizzled by row % 8)
            int b_, t0_, t1_;
            chunk_range(p.sched, u / H, b_, t0_, t1_);
            const int tq0 = t0_ / nh;
            uint4 w[8];
#pragma unroll
            for (int k8 = 0; k8 < 8; ++k8) {
                const int id = tid + kPrepThreads * k8, a = id >> 9, m = (id >> 3) & 63, j = id & 7;
                const int sr = (t0_ + m) / nh - tq0;
                w[k8] = *reinterpret_cast<const uint4*>(smem + L::OFF_QK + a * 16384 + sr * 128 + ((j ^ (sr & 7)) * 16));
            }
            __syncthreads();
#pragma unroll
            for (int k8 = 0; k8 < 8; ++k8) {
                const int id = tid + kPrepThreads * k8, a = id >> 9, m = (id >> 3) & 63, j = id & 7;
                *reinterpret_cast<uint4*>(smem + L::OFF_QK + a * 16384 + m * 128 + ((j ^ (m & 7)) * 16)) = w[k8];
            }
            sm100::fence_async_smem();
            __syncthreads();
        }
        if constexpr (GATED) {
            // running sums c_l of the chunk's log decays (read after the next barrier)
            if (warp == 1) {
                const float2 c = gate_prefix(reinterpret_cast<const float*>(smem + L::OFF_G) + bb * kChunk, 1, 0,
                                             kChunk);
                reinterpret_cast<float2*>(smem + L::OFF_C)[lane] = c;
                reinterpret_cast<float2*>(smem + L::OFF_LAM)[lane] = make_float2(expf(c.x), expf(c.y));
                // row factors F of the unit: lambda[l+1:C] per row, then lambda[1:C]
                const float cC = __shfl_sync(0xffffffffu, c.y, 31);
                float* F = reinterpret_cast<float*>(p.wsT + (size_t)u * kUnit + kUnitF);
                reinterpret_cast<float2*>(F)[lane] = make_float2(expf(cC - c.x), expf(cC - c.y));
                if (lane == 0) F[kChunk] = expf(cC);
            }
        }
        // G = [Q; K] K^T into 64 tensor-memory columns: lanes 0-63 Q K^T, 64-127 K K^T
        if (tid == 0) {
            sm100::tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint64_t o = (uint64_t)(((j >> 2) * 16384 + (j & 3) * 32) >> 4);
                sm100::umma_bf16(tmem, dQK + o, dQK + o + (8192 >> 4), i_g, j > 0);
            }
            sm100::umma_commit(&bars[1]);
        }
        const bool gdone = sm100::mbar_wait(&bars[1], it_ & 1, abort_flag);
        // the product has read the q/k tile: the region now takes the solve's blocks
        if (__syncthreads_or(!gdone)) break;
        sm100::tc_fence_after();
        if constexpr (GATED) {
            // Q<- = diag(lambda[1:l]) Q: the unit's two q boxes (128-byte rows, swizzled
            // within the row) scaled per token row in place and copied out unchanged in
            // layout by two bulk stores, whose reads complete before the solve's blocks
            // overwrite the region (asynchronous copies: no ordinary global store is left in
            // flight ahead of the tensor-memory reads below)
            const float* lam = reinterpret_cast<const float*>(smem + L::OFF_LAM);
#pragma unroll
            for (int k8 = 0; k8 < 8; ++k8) {
                const int id = tid + kPrepThreads * k8, a = id >> 9, row = (id >> 3) & 63, pc = id & 7;
                uint4* ptr = reinterpret_cast<uint4*>(smem + L::OFF_QK + a * 16384 + row * 128 + pc * 16);
                const float f = lam[row];
                uint4 v = *ptr;
                v.x = scale_pair(v.x, f);
                v.y = scale_pair(v.y, f);
                v.z = scale_pair(v.z, f);
                v.w = scale_pair(v.w, f);
                *ptr = v;
            }
            sm100::fence_async_smem();
            __syncthreads();
            if (tid == 0) {
                uint8_t* dst = p.wsT + (size_t)u * kUnit + kUnitQL;
                sm100::bulk_store(dst, smem + L::OFF_QK, 8192);
                sm100::bulk_store(dst + 8192, smem + L::OFF_QK + 16384, 8192);
                sm100::bulk_commit();
                sm100::bulk_wait_read0();
            }
            __syncthreads();
            DN_TRP(it_, 6);
        }
        const float* betas = reinterpret_cast<const float*>(smem + L::OFF_BETA) + bb * kChunk;
        const float* cs = reinterpret_cast<const float*>(smem + L::OFF_C);  // gated: running sums
        {
            const int i = 32 * (warp & 1) + lane;  // row of Q K^T (warps 0, 1) or K K^T (warps 2, 3)
            const uint32_t taddr = tmem + ((uint32_t)(32 * warp) << 16);
            // gated: Gamma[i][j] = exp(c_i - c_j) for j <= i (c falls with j, so <= 1)
            const float ci = GATED ? cs[i] : 0.f;
            auto gam = [&](int j) -> float {
                if constexpr (GATED) return __expf(ci - cs[j]);
                else return 1.f;
            };
            if (warp >= 2) {
                // A = B L, blocked: row i of block row bi; blocks left of the diagonal
                // row-major, the diagonal block transposed (for the column sweeps)
                const int bi = i >> 4, ri = i & 15;
                const float bta = betas[i];
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {
                    uint32_t v[32];
                    sm100::tmem_ld32(taddr + 32 * hc, v);
#pragma unroll
                    for (int bh = 0; bh < 2; ++bh) {
                        const int bj = 2 * hc + bh;
                        if (bj > bi) continue;
                        float* blk = Ablk + blk_index(bi, bj) * kBlkFloats;
                        if (bj < bi) {
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4) {
                                const int j = 16 * bj + 4 * q4;
                                float4 f;
                                f.x = bta * gam(j) * __uint_as_float(v[16 * bh + 4 * q4 + 0]);
                                f.y = bta * gam(j + 1) * __uint_as_float(v[16 * bh + 4 * q4 + 1]);
                                f.z = bta * gam(j + 2) * __uint_as_float(v[16 * bh + 4 * q4 + 2]);
                                f.w = bta * gam(j + 3) * __uint_as_float(v[16 * bh + 4 * q4 + 3]);
                                *reinterpret_cast<float4*>(blk + ri * kBlkLd + 4 * q4) = f;
                            }
                        } else {
#pragma unroll
                            for (int c = 0; c < 16; ++c)
                                blk[c * kBlkLd + ri] =
                                    c < ri ? bta * gam(16 * bj + c) * __uint_as_float(v[16 * bh + c]) : 0.f;
                        }
                    }
                }
            } else {
                // P = (Q K^T) o M_c, inclusive: bf16 row i of the unit's P tile, staged
                // where the N blocks are written after the diagonal solve
                uint8_t* ps = smem + L::OFF_N;
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {
                    uint32_t v[32];
                    sm100::tmem_ld32(taddr + 32 * hc, v);
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        const int col = 32 * hc + 8 * c8;
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            x[e] = (col + e <= i) ? gam(col + e) * __uint_as_float(v[8 * c8 + e]) : 0.f;
                        uint4 w;
                        w.x = sm100::pack_bf16(x[0], x[1]);
                        w.y = sm100::pack_bf16(x[2], x[3]);
                        w.z = sm100::pack_bf16(x[4], x[5]);
                        w.w = sm100::pack_bf16(x[6], x[7]);
                        *reinterpret_cast<uint4*>(ps + sm100::swz128(i, col)) = w;
                    }
                }
                DN_TRP(it_, 7);
                sm100::fence_async_smem();
            }
        }
        sm100::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            sm100::bulk_store(p.wsT + (size_t)u * kUnit + 8192, smem + L::OFF_N, 8192);
            sm100::bulk_commit();
        }
        DN_TRP(it_, 2);
        // diagonal block `warp` of N = (I + A)^{-1}: one column per lane (lanes 16-31
        // repeat 0-15), right-looking: once x_j is final it updates every later row.
        // Column j + 1 of A (contiguous: the block is stored transposed) is loaded
        // with four 16-byte loads while column j is applied.
        {
            const int c = lane & 15;
            const float* At = Ablk + blk_index(warp, warp) * kBlkFloats;  // At[j][i] = A[i][j]
            float x[16], cur[16], nxt[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = (i == c) ? 1.f : 0.f;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float4 f = *reinterpret_cast<const float4*>(At + 4 * q4);
                cur[4 * q4] = f.x; cur[4 * q4 + 1] = f.y; cur[4 * q4 + 2] = f.z; cur[4 * q4 + 3] = f.w;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (j + 1 < 16) {
#pragma unroll
                    for (int q4 = (j + 2) / 4; q4 < 4; ++q4) {
                        const float4 f = *reinterpret_cast<const float4*>(At + (j + 1) * kBlkLd + 4 * q4);
                        nxt[4 * q4] = f.x; nxt[4 * q4 + 1] = f.y; nxt[4 * q4 + 2] = f.z; nxt[4 * q4 + 3] = f.w;
                    }
                }
#pragma unroll
                for (int i = j + 1; i < 16; ++i) x[i] = fmaf(-cur[i], x[j], x[i]);
#pragma unroll
                for (int i = j + 2; i < 16; ++i) cur[i] = nxt[i];
            }
            // the P copy has read its staging, which the N blocks overwrite
            if (tid == 0) sm100::bulk_wait_read0();
            __syncthreads();
            if (lane < 16) {
                float* Nb = Nblk + blk_index(warp, warp) * kBlkFloats;
#pragma unroll
                for (int i = 0; i < 16; ++i) Nb[i * kBlkLd + c] = x[i];
            }
        }
        __syncthreads();
        DN_TRP(it_, 3);
        // off-diagonal blocks N_ij = -N_ii sum_{k=j}^{i-1} A_ik N_kj; the products that
        // do not depend on earlier results run first, spread over the four warps
        {
            auto A_ = [&](int i, int j) { return Ablk + blk_index(i, j) * kBlkFloats; };
            auto N_ = [&](int i, int j) { return Nblk + blk_index(i, j) * kBlkFloats; };
            float* X = Xs + warp * kBlkFloats;          // per-warp staging (warps 0-2)
            float* Y20 = Xs + 3 * kBlkFloats;           // shared partial sums
            float* Y31 = Xs + 4 * kBlkFloats;
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            float y30[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            // phase 1: N_{i+1,i} for i = 0, 1, 2 (warps 0-2); warp 3: A20 N00 and A31 N11
            if (warp < 3) {
                mm16_tf32(acc, A_(warp + 1, warp), N_(warp, warp));
                finish_block(Nblk, X, warp + 1, warp, acc);
            } else {
                mm16_tf32(acc, A_(2, 0), N_(0, 0));
                st_blk(Y20, acc, 1.f);
                float a2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                mm16_tf32(a2, A_(3, 1), N_(1, 1));
                st_blk(Y31, a2, 1.f);
            }
            __syncthreads();
            // phase 2: N20 (warp 0), N31 (warp 1), and A30 N00 + A31 N10 (warp 2)
            if (warp == 0) {
                ld_blk(acc, Y20);
                mm16_tf32(acc, A_(2, 1), N_(1, 0));
                finish_block(Nblk, X, 2, 0, acc);
            } else if (warp == 1) {
                ld_blk(acc, Y31);
                mm16_tf32(acc, A_(3, 2), N_(2, 1));
                finish_block(Nblk, X, 3, 1, acc);
            } else if (warp == 2) {
                mm16_tf32(y30, A_(3, 0), N_(0, 0));
                mm16_tf32(y30, A_(3, 1), N_(1, 0));
            }
            __syncthreads();
            // phase 3: N30 (warp 2)
            if (warp == 2) {
                mm16_tf32(y30, A_(3, 2), N_(2, 0));
                finish_block(Nblk, X, 3, 0, y30);
            }
            // gated: the previous unit's T' copy has read its staging, rewritten below
            if (GATED && tid == 0) sm100::bulk_wait_read0();
            __syncthreads();
        }
        DN_TRP(it_, 4);
        // T = N diag(beta) -> bf16 tile (128-byte rows, 128-byte swizzle), built where
        // the A blocks were and copied out in one piece.  Thread: row i (consecutive
        // over a warp's lanes, so that a quarter-warp's 16-byte accesses fall into 8
        // distinct bank groups), half hh of the columns.
        {
            const int i = 32 * (warp & 1) + lane, hh = warp >> 1, bi = i >> 4;
            uint8_t* tg = smem + L::OFF_A;
            uint4 t2w[4];  // gated: this thread's pieces of T', written once N is read
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int j0 = 32 * hh + 8 * cc, bj = j0 >> 4;
                const float4 b0 = *reinterpret_cast<const float4*>(betas + j0);
                const float4 b1 = *reinterpret_cast<const float4*>(betas + j0 + 4);
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                float vals[8];
                (void)cs;
                if (bj <= bi) {
                    const float* nr = Nblk + blk_index(bi, bj) * kBlkFloats + (i & 15) * kBlkLd + (j0 & 15);
                    const float4 f0 = *reinterpret_cast<const float4*>(nr);
                    const float4 f1 = *reinterpret_cast<const float4*>(nr + 4);
                    const float nv[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) vals[e] = (j0 + e <= i) ? nv[e] * bv[e] : 0.f;
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) vals[e] = 0.f;
                }
                uint4 w;
                w.x = sm100::pack_bf16(vals[0], vals[1]);
                w.y = sm100::pack_bf16(vals[2], vals[3]);
                w.z = sm100::pack_bf16(vals[4], vals[5]);
                w.w = sm100::pack_bf16(vals[6], vals[7]);
                *reinterpret_cast<uint4*>(tg + sm100::swz128(i, j0)) = w;
                if constexpr (GATED) {
                    // T' = T diag(lambda[1:j]), lambda[1:j] = exp(c_j) <= 1
                    const float* lam = reinterpret_cast<const float*>(smem + L::OFF_LAM);
                    float l8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) l8[e] = vals[e] * lam[j0 + e];
                    t2w[cc].x = sm100::pack_bf16(l8[0], l8[1]);
                    t2w[cc].y = sm100::pack_bf16(l8[2], l8[3]);
                    t2w[cc].z = sm100::pack_bf16(l8[4], l8[5]);
                    t2w[cc].w = sm100::pack_bf16(l8[6], l8[7]);
                }
            }
            if constexpr (GATED) {
                __syncthreads();  // N is read: T' takes the region's second 8 KB
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
                    *reinterpret_cast<uint4*>(smem + L::OFF_T2 + sm100::swz128(i, 32 * hh + 8 * cc)) = t2w[cc];
            }
            sm100::fence_async_smem();
        }
        __syncthreads();
        // copy T out; the region takes the next unit's q/k tile (the box over the T
        // staging once the copy has read it)
        const int un = u + gridDim.x;
        if (tid == 0) {
            sm100::bulk_store(p.wsT + (size_t)u * kUnit, smem + L::OFF_A, 8192);
            if constexpr (GATED) sm100::bulk_store(p.wsT + (size_t)u * kUnit + kUnitT2, smem + L::OFF_T2, 8192);
            sm100::bulk_commit();
        }
        if (un < units) {
            issue(un, bb ^ 1, true);
            in_flight = true;
        }
        DN_TRP(it_, 5);
    }
    // a load issued for a unit this CTA then gave up on must land before exit
    if (in_flight) {
        volatile int drain = 0;
        sm100::mbar_wait(&bars[0], it_ & 1, &drain, sm100::kDrainWaitNs);
    }
    cp_async_wait<0>();
    if (tid == 0) {
        sm100::bulk_wait0();             // the tile copies are complete
        sm100::umma_drain(&bars[2]);     // and the last Gram product (a wait for it may have given up)
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, 64);
    }
    if (tid == 0 && *abort_flag) atomicExch(p.err, kErrTimeout);
}

}  // namespace dn
