// UT pre-pass: the chunk-local factor of every (chunk, head), computed once.
//
// "Context Parallelism for DeltaNet", section 2, step 1: the WY factors of a
// chunk depend only on that chunk's keys and step sizes, so every chunk can be
// processed in parallel.  Per (chunk r, head) this kernel forms
//   L_r = (K_r K_r^T) o M_c^-,    T_r = (I + B_r L_r)^{-1} B_r
// ("Linear Attention, Visualized", DeltaNet, "Complete per-chunk algorithm")
// and stores T_r as a bf16 64 x 64 tile whose rows are 128 bytes with the
// 128-byte swizzle, i.e. exactly the shared-memory layout in which the chain
// kernel uses T^T as a tensor-core operand (it copies the tile in with one
// bulk copy).  W_r = T_r K_r and U_r = T_r V_r are formed later, on the
// tensor cores, next to the state chain.
//
// The 64 x 64 solve is blocked in 16 x 16 blocks: N = (I + A)^{-1} with
// A = B L; each diagonal block by forward substitution (one warp per block,
// one column per lane, fp32), then N_ij = -N_ii sum_{k=j}^{i-1} A_ik N_kj in
// order of i - j with tf32 mma.sync, and T = N B.
// One CTA of 4 warps per (chunk, head) at a time, several CTAs per SM, so the
// latency of the solve is hidden by parallelism across chunks.
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
constexpr int kBlkLd = 20;  // fp32 16 x 16 blocks, 16-byte aligned rows
constexpr int kBlkFloats = 16 * kBlkLd;

template <int DK>
struct PrepSmem {
    static constexpr int K_BYTES = kChunk * DK * 2;  // one K tile; the A blocks reuse it
    static constexpr int A_BYTES = 10 * kBlkFloats * 4;
    static_assert(A_BYTES <= K_BYTES, "A blocks must fit in a K tile");
    static constexpr int OFF_K = 0;                  // 2 K tiles (double buffer)
    static constexpr int OFF_N = 2 * K_BYTES;
    static constexpr int OFF_X = OFF_N + 10 * kBlkFloats * 4;
    static constexpr int OFF_BETA = OFF_X + 6 * kBlkFloats * 4;
    static constexpr int TOTAL = OFF_BETA + 2 * kChunk * 4;
};

__device__ __forceinline__ int blk_index(int bi, int bj) { return bi * (bi + 1) / 2 + bj; }

// acc (16 x 16, two n8 tiles) += A (16 x 16) * B (16 x 16), tf32 inputs, fp32 accumulate.
__device__ __forceinline__ void mm16_tf32(float (&acc)[2][4], const float* A, const float* B) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a0 = sm100::to_tf32(A[g * kBlkLd + 8 * ks + t]);
        const uint32_t a1 = sm100::to_tf32(A[(g + 8) * kBlkLd + 8 * ks + t]);
        const uint32_t a2 = sm100::to_tf32(A[g * kBlkLd + 8 * ks + t + 4]);
        const uint32_t a3 = sm100::to_tf32(A[(g + 8) * kBlkLd + 8 * ks + t + 4]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b0 = sm100::to_tf32(B[(8 * ks + t) * kBlkLd + 8 * nt + g]);
            const uint32_t b1 = sm100::to_tf32(B[(8 * ks + t + 4) * kBlkLd + 8 * nt + g]);
            sm100::mma_tf32(acc[nt], a0, a1, a2, a3, b0, b1);
        }
    }
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

template <int DK>
__global__ void __launch_bounds__(kPrepThreads, 4) k_ut_prep(Params p) {
    using L = PrepSmem<DK>;
    extern __shared__ __align__(128) char smem[];
    float* Nblk = reinterpret_cast<float*>(smem + L::OFF_N);
    float* Xs = reinterpret_cast<float*>(smem + L::OFF_X);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    const int H = p.sched.H;
    const int units = count_chunks(p.sched) * H;

    // K tile and step sizes of unit u into buffer `buf` (cp.async; one group)
    auto issue = [&](int u, int buf) {
        const int id = u / H, head = u % H;
        int b, t0, t1;
        chunk_range(p.sched, id, b, t0, t1);
        const int rows = t1 - t0;
        const __nv_bfloat16* kg =
            static_cast<const __nv_bfloat16*>(p.k) + b * p.k_sb + head * p.k_sh + (int64_t)t0 * p.k_st;
        load_tile<__nv_bfloat16, DK, kPrepThreads>(
            reinterpret_cast<__nv_bfloat16*>(smem + L::OFF_K + buf * L::K_BYTES), kg, p.k_st, rows);
        if (tid < kChunk) {
            const bool ok = tid < rows;
            const float* src = p.beta + b * p.b_sb + (int64_t)(t0 + (ok ? tid : 0)) * p.b_st + head * p.b_sh;
            cp_async4(smem_addr(smem + L::OFF_BETA + (buf * kChunk + tid) * 4), src, ok ? 4 : 0);
        }
        cp_async_commit();
    };

    int buf = 0, it_ = 0;
    if ((int)blockIdx.x < units) issue(blockIdx.x, 0);
    for (int u = blockIdx.x; u < units; u += gridDim.x, buf ^= 1, ++it_) {
        DN_TRP(it_, 0);
        const int un = u + gridDim.x;
        if (un < units) {
            issue(un, buf ^ 1);  // prefetch the next unit while this one is computed
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        DN_TRP(it_, 1);
        __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smem + L::OFF_K + buf * L::K_BYTES);
        float* Ablk = reinterpret_cast<float*>(Ks);
        const float* betas = reinterpret_cast<const float*>(smem + L::OFF_BETA) + buf * kChunk;

        // A = B L, blocked: warp w owns rows 16w .. 16w + 15 (row block w) and only the
        // column blocks 0 .. w.  Diagonal blocks are stored transposed (column-major)
        // for the column sweeps of the solve; the others row-major for the MMAs.
        {
            float acc[8][4];
            zero_frag(acc);
            switch (warp) {
                case 0: warp_gemm<DK, 2, DK, false, DK, false>(*reinterpret_cast<float(*)[2][4]>(acc), Ks, 0, Ks, 0); break;
                case 1: warp_gemm<DK, 4, DK, false, DK, false>(*reinterpret_cast<float(*)[4][4]>(acc), Ks, 16, Ks, 0); break;
                case 2: warp_gemm<DK, 6, DK, false, DK, false>(*reinterpret_cast<float(*)[6][4]>(acc), Ks, 32, Ks, 0); break;
                default: warp_gemm<DK, 8, DK, false, DK, false>(acc, Ks, 48, Ks, 0); break;
            }
            const float b_lo = betas[16 * warp + g8], b_hi = betas[16 * warp + g8 + 8];
            __syncthreads();  // K is no longer read: its space now holds A
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int bj = nt >> 1;
                if (bj <= warp) {
                    float* blk = Ablk + blk_index(warp, bj) * kBlkFloats;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int row = 16 * warp + g8 + 8 * (e >> 1);
                        const int col = 8 * nt + 2 * t4 + (e & 1);
                        const float val = col < row ? ((e >> 1) ? b_hi : b_lo) * acc[nt][e] : 0.f;
                        if (bj == warp) blk[(col & 15) * kBlkLd + (row & 15)] = val;
                        else blk[(row & 15) * kBlkLd + (col & 15)] = val;
                    }
                }
            }
        }
        __syncthreads();
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
            float* X = Xs + warp * kBlkFloats;          // per-warp staging
            float* Y20 = Xs + 4 * kBlkFloats;           // shared partial sums
            float* Y31 = Xs + 5 * kBlkFloats;
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
            __syncthreads();
        }
        DN_TRP(it_, 4);
        // T = N diag(beta) -> bf16 tile (128-byte rows, 128-byte swizzle) in global memory
        {
            const int i = tid >> 1, hh = tid & 1, bi = i >> 4;
            uint8_t* tg = p.wsT + (size_t)u * 8192;
            float bj32[32];
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
                const float4 f = *reinterpret_cast<const float4*>(betas + 32 * hh + 4 * q4);
                bj32[4 * q4] = f.x; bj32[4 * q4 + 1] = f.y; bj32[4 * q4 + 2] = f.z; bj32[4 * q4 + 3] = f.w;
            }
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int j0 = 32 * hh + 8 * cc, bj = j0 >> 4;
                float vals[8];
                if (bj <= bi) {
                    const float* nr = Nblk + blk_index(bi, bj) * kBlkFloats + (i & 15) * kBlkLd + (j0 & 15);
                    const float4 f0 = *reinterpret_cast<const float4*>(nr);
                    const float4 f1 = *reinterpret_cast<const float4*>(nr + 4);
                    const float nv[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) vals[e] = (j0 + e <= i) ? nv[e] * bj32[8 * cc + e] : 0.f;
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
            }
        }
        __syncthreads();
    }
}

}  // namespace dn
