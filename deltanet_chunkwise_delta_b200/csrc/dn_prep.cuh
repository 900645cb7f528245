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

constexpr int kPrepThreads = 128;
constexpr int kBlkLd = 20;  // fp32 16 x 16 blocks, 16-byte aligned rows
constexpr int kBlkFloats = 16 * kBlkLd;

template <int DK>
struct PrepSmem {
    static constexpr int K_BYTES = kChunk * DK * 2;
    static constexpr int A_BYTES = 10 * kBlkFloats * 4;
    static constexpr int OFF_A = 0;  // the A blocks replace K once the Gram matrix is in registers
    static constexpr int OFF_N = (K_BYTES > A_BYTES ? K_BYTES : A_BYTES);
    static constexpr int OFF_X = OFF_N + 10 * kBlkFloats * 4;
    static constexpr int OFF_BETA = OFF_X + 4 * kBlkFloats * 4;
    static constexpr int TOTAL = OFF_BETA + kChunk * 4;
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

template <int DK>
__global__ void __launch_bounds__(kPrepThreads) k_ut_prep(Params p) {
    using L = PrepSmem<DK>;
    extern __shared__ __align__(128) char smem[];
    __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smem);
    float* Ablk = reinterpret_cast<float*>(smem + L::OFF_A);
    float* Nblk = reinterpret_cast<float*>(smem + L::OFF_N);
    float* Xs = reinterpret_cast<float*>(smem + L::OFF_X);
    float* betas = reinterpret_cast<float*>(smem + L::OFF_BETA);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    const int H = p.sched.H;
    const int units = count_chunks(p.sched) * H;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int id = u / H, head = u % H;
        int b, t0, t1;
        chunk_range(p.sched, id, b, t0, t1);
        const int rows = t1 - t0;
        const __nv_bfloat16* kg =
            static_cast<const __nv_bfloat16*>(p.k) + b * p.k_sb + head * p.k_sh + (int64_t)t0 * p.k_st;
        load_tile<__nv_bfloat16, DK, kPrepThreads>(Ks, kg, p.k_st, rows);
        cp_async_commit();
        if (tid < kChunk)
            betas[tid] = tid < rows ? p.beta[b * p.b_sb + (int64_t)(t0 + tid) * p.b_st + head * p.b_sh] : 0.f;
        cp_async_wait<0>();
        __syncthreads();

        // A = B L, blocked: warp w owns rows 16w .. 16w + 15 (row block w), columns < 16w + 16
        {
            float acc[8][4];
            zero_frag(acc);
            warp_gemm<DK, 8, DK, false, DK, false>(acc, Ks, 16 * warp, Ks, 0);
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
                        blk[(row & 15) * kBlkLd + (col & 15)] = col < row ? betas[row] * acc[nt][e] : 0.f;
                    }
                }
            }
        }
        __syncthreads();
        // diagonal block `warp` of N: one column per lane (lanes 16-31 repeat 0-15)
        {
            const int c = lane & 15;
            const float* Ab = Ablk + blk_index(warp, warp) * kBlkFloats;
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float a[16];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    if (4 * c4 < i) {
                        const float4 f = *reinterpret_cast<const float4*>(Ab + i * kBlkLd + 4 * c4);
                        a[4 * c4 + 0] = f.x;
                        a[4 * c4 + 1] = f.y;
                        a[4 * c4 + 2] = f.z;
                        a[4 * c4 + 3] = f.w;
                    }
                }
                // two partial sums shorten the dependent chain
                float s0 = (i == c) ? 1.f : 0.f, s1 = 0.f;
#pragma unroll
                for (int j = 0; j < i; ++j) {
                    if (j & 1) s1 = fmaf(-a[j], x[j], s1);
                    else s0 = fmaf(-a[j], x[j], s0);
                }
                x[i] = s0 + s1;
            }
            if (lane < 16) {
                float* Nb = Nblk + blk_index(warp, warp) * kBlkFloats;
#pragma unroll
                for (int i = 0; i < 16; ++i) Nb[i * kBlkLd + c] = x[i];
            }
        }
        __syncthreads();
        // off-diagonal blocks, by distance i - j
#pragma unroll 1
        for (int dd = 1; dd < 4; ++dd) {
            if (warp < 4 - dd) {
                const int i = warp + dd, j = warp;
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                for (int kb = j; kb < i; ++kb)
                    mm16_tf32(acc, Ablk + blk_index(i, kb) * kBlkFloats, Nblk + blk_index(kb, j) * kBlkFloats);
                float* X = Xs + warp * kBlkFloats;
                st_blk(X, acc, 1.f);
                __syncwarp();
                float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                mm16_tf32(acc2, Nblk + blk_index(i, i) * kBlkFloats, X);
                st_blk(Nblk + blk_index(i, j) * kBlkFloats, acc2, -1.f);
            }
            __syncthreads();
        }
        // T = N diag(beta) -> bf16 tile (128-byte rows, 128-byte swizzle) in global memory
        {
            const int i = tid >> 1, hh = tid & 1, bi = i >> 4;
            uint8_t* tg = p.wsT + (size_t)u * 8192;
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
                    for (int e = 0; e < 8; ++e) vals[e] = (j0 + e <= i) ? nv[e] * betas[j0 + e] : 0.f;
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
