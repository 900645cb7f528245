// One CTA threads the chunk state through a run of chunks of one (sequence, head).
//
// Per chunk r ("Linear Attention, Visualized", DeltaNet, "Complete per-chunk
// algorithm"), with B_r = diag(beta_r):
//   L_r = (K_r K_r^T) o M_c^-           strict-lower Gram matrix
//   (I + B_r L_r) T_r = B_r             UT triangular solve (blocked, fp32)
//   W_r = T_r K_r,  U_r = T_r V_r        WY / UT factors
//   Z_r = U_r - W_r S_r                  corrected writes
//   O_r = Q_r S_r + (Q_r K_r^T o M_c) Z_r
//   S_{r+1} = S_r + K_r^T Z_r
// The same loop with other start states and without output produces the
// segment maps used for context parallelism (see SegMode): the zero-start
// local writes H (V present, S_0 = 0) and the transition product P (no V,
// S_0 = I, so each chunk applies I - K_r^T W_r, subsection "Compact the
// transition product with WY").
//
// Gated DeltaNet (same page, section "Gated DeltaNet (GDN)", its "Complete
// per-chunk algorithm") adds a per-token decay a_t = exp(g_t).  With
// lambda[i:j] = a_i ... a_j inside the chunk and Gamma[l][i] = lambda[i+1:l]:
//   L_r = (K_r K_r^T o Gamma) o M_c^-,  (I + B_r L_r) T_r = B_r,  U_r = T_r V_r
//   W<-_r = T_r diag(lambda[1:l]) K_r,  Z_r = U_r - W<-_r S_r
//   O_r = diag(lambda[1:l]) Q_r S_r + (Q_r K_r^T o Gamma) Z_r
//   S_{r+1} = lambda[1:C] S_r + (diag(lambda[l+1:C]) K_r)^T Z_r
// Decay products are exponentials of differences of the chunk's running sum of
// g (fp32), so none of them is formed as a ratio of small numbers.  The left
// factor of W is folded into a second copy of T (columns scaled), the right
// factor of the state update into K (rows scaled in place once its other uses
// are done), the readout factor into the rows of Q S, and lambda[1:C] into the
// state registers.
//
// Kimi Delta Attention (same page, section "Kimi Delta Attention (KDA)", its
// complete per-chunk algorithm) decays every key channel c by its own a_t[c] =
// exp(g_t[c]).  With G_l = g_1 + ... + g_l (per channel, within the chunk):
//   L[l][m] = sum_c k_l[c] k_m[c] exp(G_l[c] - G_m[c])  (m < l),  A[l][m] the same
//   with q_l (m <= l);  (I + B_r L) T_r = B_r,  U_r = T_r V_r,  W_r = T_r K<-_r,
//   Z_r = U_r - W_r S_r,  O_r = Q<-_r S_r + A Z_r,  S_{r+1} = Diag(lambda[1:C]) S_r
//   + K->_r^T Z_r,  with q<-_l = exp(G_l) o q_l, k<-_l = exp(G_l) o k_l,
//   k->_l = exp(G_C - G_l) o k_l, lambda[1:C] = exp(G_C).
// L and A are formed block by block of 16 rows against the block's first row s:
// exp(G_l - G_m) = exp(G_l - G_s) exp(G_s - G_m), so each product takes the rows
// k_l o exp(G_l - G_s) (q_l o exp(G_l - G_s)) and k_m o exp(G_s - G_m).  For rows
// before the block both factors are products of decays (at most 1 for a_t <= 1);
// inside the block the second one grows with at most 15 tokens' decay, which keeps
// it in range for |g| < 5.8 per token and channel.
//
// The state stays in registers (fp32) for the whole run; W, U, Z, T and the
// masked scores never leave shared memory.  Only q, k, v, beta are read and o
// written per chunk.  Loads of chunk r+1 are issued before chunk r is computed.
#pragma once

#include "dn_common.cuh"
#include "dn_sm100.cuh"
#include "dn_warp_gemm.cuh"

namespace dn {

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

template <typename E, int DK, int NX, bool HAS_V, bool HAS_Q, int STAGES, bool GATED = false,
          bool KDA = false>
struct ChainSmem {
    static constexpr int ES = sizeof(E);
    static constexpr int Q_BYTES = kChunk * DK * ES;
    static constexpr int K_BYTES = kChunk * DK * ES;
    static constexpr int V_BYTES = kChunk * NX * ES;
    static constexpr int SOLVE_LD = 65;  // fp32 solve tiles, padded against bank conflicts
    static constexpr int SOLVE_BYTES = (2 * kChunk * SOLVE_LD + 3 * 256) * 4;
    static constexpr int O_BYTES = HAS_Q ? kChunk * NX * ES : 0;
    static constexpr int UNION_BYTES = SOLVE_BYTES > O_BYTES ? SOLVE_BYTES : O_BYTES;

    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + (HAS_Q ? STAGES * Q_BYTES : 0);
    static constexpr int OFF_V = OFF_K + STAGES * K_BYTES;
    static constexpr int OFF_BETA = OFF_V + (HAS_V ? STAGES * V_BYTES : 0);
    // g per stage: one per token (GATED), or one per (token, key channel) as an fp32 tile
    // of 64 rows x DK, row-major (KDA; made the chunk's running sums in place)
    static constexpr int GATE_BYTES = KDA ? kChunk * DK * 4 : (GATED ? kChunk * 4 : 0);
    static constexpr int OFF_GATE = OFF_BETA + STAGES * kChunk * 4;
    static constexpr int OFF_DECAY = OFF_GATE + STAGES * GATE_BYTES;
    // GATED: running sum, lambda[1:l], lambda[l+1:C], lambda[1:C]; KDA: lambda[1:C] per channel
    static constexpr int OFF_SOLVE = OFF_DECAY + (GATED ? 4 * kChunk * 4 : (KDA ? DK * 4 : 0));
    static constexpr int OFF_T = align_up(OFF_SOLVE + UNION_BYTES, 128);
    static constexpr int OFF_W = OFF_T + kChunk * kChunk * ES;
    static constexpr int OFF_X = OFF_W + kChunk * DK * ES;
    static constexpr int OFF_Z = OFF_X + DK * NX * ES;
    static constexpr int OFF_P = OFF_Z + kChunk * NX * ES;
    static constexpr int OFF_T2 = OFF_P + (HAS_Q ? kChunk * kChunk * ES : 0);
    // KDA: scratch rows of K scaled by decay ratios (one 16-row block's operands at a time,
    // later K<-), and the block's left operands [K rows; Q rows] (2 x 16 rows)
    static constexpr int OFF_R = OFF_T2 + (GATED ? kChunk * kChunk * ES : 0);
    static constexpr int OFF_LQ = OFF_R + (KDA ? kChunk * DK * ES : 0);
    static constexpr int TOTAL = OFF_LQ + (KDA ? 2 * 16 * DK * ES : 0);
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
                 "r"(src_bytes));
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src),
                 "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// Copy a 64-row tile (row stride `st` elements in global memory) into a
// swizzled shared tile of width D; rows >= rows_valid are zero-filled.
template <typename E, int D, int NT = kThreads>
__device__ __forceinline__ void load_tile(E* dst, const E* src, int64_t st, int rows_valid) {
    constexpr int V = 16 / sizeof(E);
    constexpr int CPR = D / V;
    for (int idx = threadIdx.x; idx < kChunk * CPR; idx += NT) {
        const int r = idx / CPR, c = idx % CPR;
        const bool ok = r < rows_valid;
        const E* s = ok ? src + r * st + c * V : src;
        cp_async16(smem_addr(dst + Swz<E>::template off<D>(r, c * V)), s, ok ? 16 : 0);
    }
}

template <typename E>
__device__ __forceinline__ E to_e(float x);
template <>
__device__ __forceinline__ __nv_bfloat16 to_e<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}
template <>
__device__ __forceinline__ float to_e<float>(float x) {
    return x;
}

// 16 x 16 fp32 blocks of row stride LD as tf32 warp products (one warp):
// acc (16 x 16, two n8 tiles in the m16n8 accumulator layout) += A * B.
template <int LD>
__device__ __forceinline__ void blk16_tf32(float (&acc)[2][4], const float* A, const float* B) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a0 = sm100::to_tf32(A[g * LD + 8 * ks + t]);
        const uint32_t a1 = sm100::to_tf32(A[(g + 8) * LD + 8 * ks + t]);
        const uint32_t a2 = sm100::to_tf32(A[g * LD + 8 * ks + t + 4]);
        const uint32_t a3 = sm100::to_tf32(A[(g + 8) * LD + 8 * ks + t + 4]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b0 = sm100::to_tf32(B[(8 * ks + t) * LD + 8 * nt + g]);
            const uint32_t b1 = sm100::to_tf32(B[(8 * ks + t + 4) * LD + 8 * nt + g]);
            sm100::mma_tf32(acc[nt], a0, a1, a2, a3, b0, b1);
        }
    }
}
template <int LD>
__device__ __forceinline__ void blk16_store(float* C, const float (&acc)[2][4], float scale) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        C[g * LD + 8 * nt + 2 * t] = scale * acc[nt][0];
        C[g * LD + 8 * nt + 2 * t + 1] = scale * acc[nt][1];
        C[(g + 8) * LD + 8 * nt + 2 * t] = scale * acc[nt][2];
        C[(g + 8) * LD + 8 * nt + 2 * t + 1] = scale * acc[nt][3];
    }
}
template <int LD>
__device__ __forceinline__ void blk16_load(float (&acc)[2][4], const float* C) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        acc[nt][0] = C[g * LD + 8 * nt + 2 * t];
        acc[nt][1] = C[g * LD + 8 * nt + 2 * t + 1];
        acc[nt][2] = C[(g + 8) * LD + 8 * nt + 2 * t];
        acc[nt][3] = C[(g + 8) * LD + 8 * nt + 2 * t + 1];
    }
}
// N_ij = -N_ii Y for a finished sum Y held in acc, through the staging block X (one warp).
template <int LD>
__device__ __forceinline__ void blk16_finish(float* Nij, const float* Nii, float* X, const float (&acc)[2][4]) {
    blk16_store<LD>(X, acc, 1.f);
    __syncwarp();
    float out[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    blk16_tf32<LD>(out, Nii, X);
    blk16_store<LD>(Nij, out, -1.f);
}

// Blocked solve of (I + A) N = I for the strictly lower A (= B L, 64 x 64, fp32,
// row stride 65), followed by T = N diag(beta) written to a swizzled tile, and,
// when colscale is given, T diag(colscale) to a second tile T2.
// Diagonal 16 x 16 blocks by forward substitution, one warp per block and one column per
// lane (lanes 16-31 repeat 0-15: two blocks in one warp would sit 16 * 65 + 16 floats apart,
// in the same banks); off-diagonal blocks by N_ij = -N_ii sum_{k=j}^{i-1} A_ik N_kj, in order
// of i - j.  N's strictly upper blocks are never read as N.  For bf16 operands (whose T is
// rounded to bf16 anyway) the off-diagonal block products take tf32 inputs on the tensor
// cores, one warp per block, staged in those upper blocks; fp32 runs them as fp32 FMAs.
template <typename E, int NT = kThreads>
__device__ __forceinline__ void ut_solve(const float* Af, float* Nf, float* Xt,
                                         const float* beta, E* Ts,
                                         const float* colscale = nullptr, E* T2 = nullptr) {
    static_assert(NT >= 128, "one warp per diagonal block");
    constexpr int LD = 65;
    const int tid = threadIdx.x;
    if (tid < 128) {
        const int blk = tid >> 5, c = tid & 15;
        const float* Ab = Af + (16 * blk) * LD + 16 * blk;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float a = (i == c) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) a = fmaf(-Ab[i * LD + j], x[j], a);
            x[i] = a;
        }
        if ((tid & 31) < 16) {
            float* Nb = Nf + (16 * blk) * LD + 16 * blk;
#pragma unroll
            for (int i = 0; i < 16; ++i) Nb[i * LD + c] = x[i];
        }
    }
    __syncthreads();
    if constexpr (std::is_same<E, __nv_bfloat16>::value) {
        const int warp = tid >> 5;
        auto A_ = [&](int i, int j) { return Af + (16 * i) * LD + 16 * j; };
        auto N_ = [&](int i, int j) { return Nf + (16 * i) * LD + 16 * j; };
        auto U_ = [&](int u) {  // staging: the strictly upper blocks (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
            const int bi = u < 3 ? 0 : (u < 5 ? 1 : 2), bj = u < 3 ? u + 1 : (u < 5 ? u - 1 : 3);
            return Nf + (16 * bi) * LD + 16 * bj;
        };
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        float y30[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        // N_{i+1,i} (warps 0-2); warp 3: the partial sums A20 N00 and A31 N11
        if (warp < 3) {
            blk16_tf32<LD>(acc, A_(warp + 1, warp), N_(warp, warp));
            blk16_finish<LD>(N_(warp + 1, warp), N_(warp + 1, warp + 1), U_(warp), acc);
        } else if (warp == 3) {
            blk16_tf32<LD>(acc, A_(2, 0), N_(0, 0));
            blk16_store<LD>(U_(3), acc, 1.f);
            float a2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            blk16_tf32<LD>(a2, A_(3, 1), N_(1, 1));
            blk16_store<LD>(U_(4), a2, 1.f);
        }
        __syncthreads();
        // N20 (warp 0), N31 (warp 1); warp 2: A30 N00 + A31 N10
        if (warp == 0) {
            blk16_load<LD>(acc, U_(3));
            blk16_tf32<LD>(acc, A_(2, 1), N_(1, 0));
            blk16_finish<LD>(N_(2, 0), N_(2, 2), U_(0), acc);
        } else if (warp == 1) {
            blk16_load<LD>(acc, U_(4));
            blk16_tf32<LD>(acc, A_(3, 2), N_(2, 1));
            blk16_finish<LD>(N_(3, 1), N_(3, 3), U_(1), acc);
        } else if (warp == 2) {
            blk16_tf32<LD>(y30, A_(3, 0), N_(0, 0));
            blk16_tf32<LD>(y30, A_(3, 1), N_(1, 0));
        }
        __syncthreads();
        // N30 (warp 2)
        if (warp == 2) {
            blk16_tf32<LD>(y30, A_(3, 2), N_(2, 0));
            blk16_finish<LD>(N_(3, 0), N_(3, 3), U_(2), y30);
        }
        __syncthreads();
    } else {
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
        const int npairs = 4 - d;
        for (int e = tid; e < npairs * 256; e += NT) {
            const int p = e >> 8, i = d + p, j = p, ri = (e >> 4) & 15, cj = e & 15;
            float acc = 0.f;
            for (int kb = j; kb < i; ++kb) {
                const float* Ar = Af + (16 * i + ri) * LD + 16 * kb;
                const float* Nc = Nf + (16 * kb) * LD + 16 * j + cj;
#pragma unroll
                for (int m = 0; m < 16; ++m) acc = fmaf(Ar[m], Nc[m * LD], acc);
            }
            Xt[p * 256 + ri * 16 + cj] = acc;
        }
        __syncthreads();
        for (int e = tid; e < npairs * 256; e += NT) {
            const int p = e >> 8, i = d + p, j = p, ri = (e >> 4) & 15, cj = e & 15;
            const float* Nr = Nf + (16 * i + ri) * LD + 16 * i;
            float acc = 0.f;
            for (int m = 0; m <= ri; ++m) acc = fmaf(Nr[m], Xt[p * 256 + m * 16 + cj], acc);
            Nf[(16 * i + ri) * LD + 16 * j + cj] = -acc;
        }
        __syncthreads();
    }
    }
    for (int e = tid; e < kChunk * kChunk; e += NT) {
        const int i = e >> 6, j = e & 63;
        const float val = j <= i ? Nf[i * LD + j] * beta[j] : 0.f;
        Ts[Swz<E>::template off<kChunk>(i, j)] = to_e<E>(val);
        if (colscale) T2[Swz<E>::template off<kChunk>(i, j)] = to_e<E>(val * colscale[j]);
    }
}

// Runs one work item.  mode selects start state, output and destination.
template <typename E, int DK, int NX, bool HAS_V, bool HAS_Q, int STAGES, bool GATED = false,
          bool KDA = false>
__device__ __forceinline__ void run_segment(const Params& p, const Item& it, int mode,
                                            char* smem) {
    using L = ChainSmem<E, DK, NX, HAS_V, HAS_Q, STAGES, GATED, KDA>;
    static_assert(!(GATED && KDA), "one kind of gate");
    using SW = Swz<E>;
    constexpr int MT_S = DK / 64;  // 16-row tiles of the state per warp
    constexpr int NT_X = NX / 16;  // 8-column tiles per warp (NX / 2 columns)
    constexpr int NT_W = DK / 16;

    E* Qs = reinterpret_cast<E*>(smem + L::OFF_Q);
    E* Ks = reinterpret_cast<E*>(smem + L::OFF_K);
    E* Vs = reinterpret_cast<E*>(smem + L::OFF_V);
    float* betas = reinterpret_cast<float*>(smem + L::OFF_BETA);
    float* gates = reinterpret_cast<float*>(smem + L::OFF_GATE);
    // per chunk (gated): running sum of g, lambda[1:l], lambda[l+1:C], lambda[1:C]
    float* gsum = reinterpret_cast<float*>(smem + L::OFF_DECAY);
    float* lam_l = gsum + kChunk;
    float* lam_r = lam_l + kChunk;
    float* lam_c = lam_r + kChunk;
    E* Ts2 = reinterpret_cast<E*>(smem + L::OFF_T2);
    // KDA: the per-channel gate tile of each stage, lambda[1:C] per channel, scratch rows
    float* gtile = reinterpret_cast<float*>(smem + L::OFF_GATE);
    float* lamc_k = reinterpret_cast<float*>(smem + L::OFF_DECAY);
    E* Rs = reinterpret_cast<E*>(smem + L::OFF_R);
    E* LQs = reinterpret_cast<E*>(smem + L::OFF_LQ);
    float* Af = reinterpret_cast<float*>(smem + L::OFF_SOLVE);
    float* Nf = Af + kChunk * L::SOLVE_LD;
    float* Xt = Nf + kChunk * L::SOLVE_LD;
    E* Os = reinterpret_cast<E*>(smem + L::OFF_SOLVE);  // aliases the solve tiles
    E* Ts = reinterpret_cast<E*>(smem + L::OFF_T);
    E* Ws = reinterpret_cast<E*>(smem + L::OFF_W);
    E* Xb = reinterpret_cast<E*>(smem + L::OFF_X);
    E* Zs = reinterpret_cast<E*>(smem + L::OFF_Z);
    E* Ps = reinterpret_cast<E*>(smem + L::OFF_P);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    const int mt = warp & 3, nh = warp >> 2;
    const int s_r0 = (DK / 4) * mt;
    const int x_c0 = (NX / 2) * nh;

    // ---- start state and destination
    const float* x_in = nullptr;
    float* x_out = nullptr;
    bool identity = false;
    const float* s0 = p.s0 ? p.s0 + it.seq * p.s0_sn + it.head * p.s0_sh : nullptr;
    if (mode == kModeOut) {
        x_in = it.g == 0 ? s0 : p.wsS + (int64_t)(it.slot + it.g - 1) * DK * NX;
        if (it.g == it.G - 1 && p.sT) x_out = p.sT + it.seq * p.sT_sn + it.head * p.sT_sh;
    } else if (mode == kModeEnd) {
        x_in = s0;
        x_out = p.wsH + (int64_t)it.slot * DK * NX;
    } else if (mode == kModeH) {
        x_out = p.wsH + (int64_t)(it.slot + it.g) * DK * NX;
    } else {
        identity = true;
        x_out = p.wsP + (int64_t)(it.slot + it.g) * DK * NX;
    }

    float s[MT_S][NT_X][4];
#pragma unroll
    for (int m = 0; m < MT_S; ++m)
#pragma unroll
        for (int nt = 0; nt < NT_X; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int r = s_r0 + 16 * m + g8 + 8 * h;
                const int c = x_c0 + 8 * nt + 2 * t4;
                float2 v2 = make_float2(0.f, 0.f);
                if (x_in) {
                    v2 = *reinterpret_cast<const float2*>(x_in + r * NX + c);
                } else if (identity) {
                    v2.x = (r == c) ? 1.f : 0.f;
                    v2.y = (r == c + 1) ? 1.f : 0.f;
                }
                s[m][nt][2 * h] = v2.x;
                s[m][nt][2 * h + 1] = v2.y;
            }

    const E* qg = static_cast<const E*>(p.q) + it.b * p.q_sb + it.head * p.q_sh;
    const E* kg = static_cast<const E*>(p.k) + it.b * p.k_sb + it.head * p.k_sh;
    const E* vg = static_cast<const E*>(p.v) + it.b * p.v_sb + it.head * p.v_sh;
    E* og = static_cast<E*>(p.o) + it.b * p.o_sb + it.head * p.o_sh;
    const float* bg = p.beta + it.b * p.b_sb + it.head * p.b_sh;
    const float* gg = (GATED || KDA) ? p.g + it.b * p.g_sb + it.head * p.g_sh : nullptr;
    // Gated Delta Product: item token ranges count virtual steps, nsub per token
    const int nsub = (GATED && p.nh > 1) ? p.nh : 1;

    const int ntok = it.tok1 - it.tok0;
    const int nchunks = (ntok + kChunk - 1) / kChunk;

    auto issue_load = [&](int r, int stg) {
        const int t0 = it.tok0 + r * kChunk;
        const int rows = min(kChunk, it.tok1 - t0);
        if (HAS_Q) {
            if (GATED && nsub > 1) {
                // the query of token m / nsub sits on its last step; other steps read zeros
                constexpr int V = 16 / sizeof(E);
                constexpr int CPR = DK / V;
                E* dst = Qs + stg * (L::Q_BYTES / L::ES);
                for (int idx = tid; idx < kChunk * CPR; idx += kThreads) {
                    const int r = idx / CPR, c = idx % CPR;
                    const int m = t0 + r;
                    const bool ok = r < rows && m % nsub == nsub - 1;
                    const E* src = ok ? qg + (int64_t)(m / nsub) * p.q_st + c * V : qg;
                    cp_async16(smem_addr(dst + SW::template off<DK>(r, c * V)), src, ok ? 16 : 0);
                }
            } else {
                load_tile<E, DK>(Qs + stg * (L::Q_BYTES / L::ES), qg + t0 * p.q_st, p.q_st, rows);
            }
        }
        load_tile<E, DK>(Ks + stg * (L::K_BYTES / L::ES), kg + t0 * p.k_st, p.k_st, rows);
        if (HAS_V) load_tile<E, NX>(Vs + stg * (L::V_BYTES / L::ES), vg + t0 * p.v_st, p.v_st, rows);
        if (tid < kChunk) {
            const bool ok = tid < rows;
            cp_async4(smem_addr(betas + stg * kChunk + tid), ok ? bg + (t0 + tid) * p.b_st : bg,
                      ok ? 4 : 0);
        }
        if constexpr (KDA) {
            // the chunk's log decays per (token, key channel): 64 rows x DK, rows past the
            // run read g = 0 (identity steps)
            float* dst = gtile + stg * (L::GATE_BYTES / 4);
            constexpr int CPR = DK / 4;
            for (int idx = tid; idx < kChunk * CPR; idx += kThreads) {
                const int rr = idx / CPR, c = idx % CPR;
                const bool ok = rr < rows;
                const float* src = ok ? gg + (int64_t)(t0 + rr) * p.g_st + 4 * c : gg;
                cp_async16(smem_addr(dst + rr * DK + 4 * c), src, ok ? 16 : 0);
            }
        }
        if (GATED && warp == 0) {
            // warp 0 loads all 64 gates (two per lane: it scans them itself after its own
            // wait, with no barrier); rows past the run read g = 0, an identity step
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // the decay of token m / nsub sits on its first step; other steps read g = 0
                const int i = 2 * lane + h;
                const int m = t0 + i;
                const bool ok = i < rows && m % nsub == 0;
                cp_async4(smem_addr(gates + stg * kChunk + i),
                          ok ? gg + (int64_t)(m / nsub) * p.g_st : gg, ok ? 4 : 0);
            }
        }
        cp_async_commit();
    };

    if (STAGES == 2 && nchunks > 0) issue_load(0, 0);

#pragma unroll 1
    for (int r = 0; r < nchunks; ++r) {
        const int stg = STAGES == 2 ? (r & 1) : 0;
        if (STAGES == 2) {
            if (r + 1 < nchunks) {
                issue_load(r + 1, stg ^ 1);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
        } else {
            issue_load(r, 0);
            cp_async_wait<0>();
        }
        const E* Qc = Qs + stg * (L::Q_BYTES / L::ES);
        const E* Kc = Ks + stg * (L::K_BYTES / L::ES);
        const E* Vc = Vs + stg * (L::V_BYTES / L::ES);
        const float* bc = betas + stg * kChunk;

        if constexpr (GATED) {
            // running sum of g over the chunk (warp scan of lane pairs) and the decay
            // products as exponentials of its differences; published by barrier (a)
            if (warp == 0) {
                const float x0 = gates[stg * kChunk + 2 * lane];
                const float x1 = gates[stg * kChunk + 2 * lane + 1];
                const float pair = x0 + x1;
                float incl = pair;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                const float c0 = (incl - pair) + x0;
                const float c1 = c0 + x1;
                const float total = __shfl_sync(0xffffffffu, c1, 31);
                gsum[2 * lane] = c0;
                gsum[2 * lane + 1] = c1;
                lam_l[2 * lane] = expf(c0);
                lam_l[2 * lane + 1] = expf(c1);
                lam_r[2 * lane] = expf(total - c0);
                lam_r[2 * lane + 1] = expf(total - c1);
                if (lane == 0) lam_c[0] = expf(total);
            }
        }

        if constexpr (HAS_Q) {
            // the state entering chunk r, for a backward pass (row = global chunk index)
            const int64_t row = (int64_t)it.cbase + r;
            if (p.cs && row < p.cs_rows) {
                float* dst = p.cs + row * p.cs_sc + it.head * p.cs_sh;
#pragma unroll
                for (int m = 0; m < MT_S; ++m)
#pragma unroll
                    for (int nt = 0; nt < NT_X; ++nt)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int rr = s_r0 + 16 * m + g8 + 8 * h;
                            const int c = x_c0 + 8 * nt + 2 * t4;
                            *reinterpret_cast<float2*>(dst + rr * NX + c) =
                                make_float2(s[m][nt][2 * h], s[m][nt][2 * h + 1]);
                        }
            }
        }

        // (a) state -> operand copy
#pragma unroll
        for (int m = 0; m < MT_S; ++m) store_frag<NT_X, NX>(Xb, s_r0 + 16 * m, x_c0, s[m], 1.f);
        __syncthreads();

        if constexpr (KDA) {
            float* G = gtile + stg * (L::GATE_BYTES / 4);
            E* Kw = const_cast<E*>(Kc);
            E* Qw = const_cast<E*>(Qc);
            // (b1) the chunk's running sums per key channel, in place, and lambda[1:C]
            for (int c = tid; c < DK; c += kThreads) {
                float acc = 0.f;
                for (int l = 0; l < kChunk; ++l) {
                    acc += G[l * DK + c];
                    G[l * DK + c] = acc;
                }
                lamc_k[c] = expf(acc);
            }
            __syncthreads();
            // (b2) rows 16 b .. 16 b + 15 of A = B L (fp32, strict lower) and of the
            // readout scores P (inclusive), against reference row s = 16 b
#pragma unroll 1
            for (int b = 0; b < 4; ++b) {
                const int s = 16 * b, ncol = s + 16;
                for (int idx = tid; idx < ncol * DK; idx += kThreads) {
                    const int m = idx / DK, c = idx % DK;
                    const int o = SW::template off<DK>(m, c);
                    Rs[o] = to_e<E>(float(Kc[o]) * expf(G[s * DK + c] - G[m * DK + c]));
                }
                for (int idx = tid; idx < 16 * DK; idx += kThreads) {
                    const int lr = idx / DK, c = idx % DK, l = s + lr;
                    const float f = expf(G[l * DK + c] - G[s * DK + c]);
                    const int o = SW::template off<DK>(l, c), ol = SW::template off<DK>(lr, c);
                    LQs[ol] = to_e<E>(float(Kc[o]) * f);
                    if (HAS_Q) LQs[16 * DK + ol] = to_e<E>(float(Qc[o]) * f);
                }
                // the block's rows right of its last column are zero in both
                for (int idx = tid; idx < 16 * (kChunk - ncol); idx += kThreads) {
                    const int row = s + idx / (kChunk - ncol), col = ncol + idx % (kChunk - ncol);
                    Af[row * L::SOLVE_LD + col] = 0.f;
                    if (HAS_Q) Ps[SW::template off<kChunk>(row, col)] = to_e<E>(0.f);
                }
                __syncthreads();
                const int ntile = b + 1;
                if (warp < (HAS_Q ? 2 : 1) * ntile) {
                    const int mat = warp / ntile, j = warp % ntile;
                    float acc[2][4];
                    zero_frag(acc);
                    warp_gemm<DK, 2, DK, false, DK, false>(acc, LQs + mat * 16 * DK, 0, Rs, 16 * j);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int row = s + g8 + 8 * (e >> 1);
                            const int col = 16 * j + 8 * nt + 2 * t4 + (e & 1);
                            if (mat == 0) Af[row * L::SOLVE_LD + col] = col < row ? bc[row] * acc[nt][e] : 0.f;
                            else acc[nt][e] = col > row ? 0.f : acc[nt][e];
                        }
                    if (mat == 1) store_frag<2, kChunk>(Ps, s, 16 * j, acc, 1.f);
                }
                __syncthreads();
            }
            // (b3) K<- = exp(G) o K into the scratch rows (the W factor); K becomes K->
            // (exp(G_C - G) o K, read by the state update) and Q becomes Q<- (exp(G) o Q)
            for (int idx = tid; idx < kChunk * DK; idx += kThreads) {
                const int l = idx / DK, c = idx % DK;
                const int o = SW::template off<DK>(l, c);
                const float gl = G[l * DK + c], gC = G[(kChunk - 1) * DK + c];
                const float kv = float(Kc[o]);
                Rs[o] = to_e<E>(kv * expf(gl));
                Kw[o] = to_e<E>(kv * expf(gC - gl));
                if (HAS_Q) Qw[o] = to_e<E>(float(Qc[o]) * expf(gl));
            }
        } else {
        // (b) A = B L (strict lower, fp32) and, with output, P = (Q K^T) o M_c
        {
            float acc[4][4];
            // Gamma[row][col] = lambda[col+1:row] on and below the diagonal (gated)
            float gam[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    gam[nt][e] = 1.f;
                    if constexpr (GATED) {
                        const int row = 16 * mt + g8 + 8 * (e >> 1);
                        const int col = 32 * nh + 8 * nt + 2 * t4 + (e & 1);
                        gam[nt][e] = col <= row ? expf(gsum[row] - gsum[col]) : 0.f;
                    }
                }
            zero_frag(acc);
            warp_gemm<DK, 4, DK, false, DK, false>(acc, Kc, 16 * mt, Kc, 32 * nh);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int row = 16 * mt + g8 + 8 * (e >> 1);
                    const int col = 32 * nh + 8 * nt + 2 * t4 + (e & 1);
                    Af[row * L::SOLVE_LD + col] =
                        col < row ? bc[row] * (acc[nt][e] * gam[nt][e]) : 0.f;
                }
            if (HAS_Q) {
                zero_frag(acc);
                warp_gemm<DK, 4, DK, false, DK, false>(acc, Qc, 16 * mt, Kc, 32 * nh);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int row = 16 * mt + g8 + 8 * (e >> 1);
                        const int col = 32 * nh + 8 * nt + 2 * t4 + (e & 1);
                        acc[nt][e] = col > row ? 0.f : acc[nt][e] * gam[nt][e];
                    }
                store_frag<4, kChunk>(Ps, 16 * mt, 32 * nh, acc, 1.f);
            }
        }
        }
        __syncthreads();

        // (c) T = (I + B L)^{-1} B
        if constexpr (GATED) ut_solve<E>(Af, Nf, Xt, bc, Ts, lam_l, Ts2);
        else ut_solve<E>(Af, Nf, Xt, bc, Ts);
        __syncthreads();

        // (d) -W = -T K (stored negated), U = T V (kept in registers as Z's start)
        float z[NT_X][4];
        zero_frag(z);
        {
            float w[NT_W][4];
            zero_frag(w);
            warp_gemm<kChunk, NT_W, kChunk, false, DK, true>(w, GATED ? Ts2 : Ts, 16 * mt,
                                                             KDA ? Rs : Kc, nh * (DK / 2));
            store_frag<NT_W, DK>(Ws, 16 * mt, nh * (DK / 2), w, -1.f);
            if (HAS_V) warp_gemm<kChunk, NT_X, kChunk, false, NX, true>(z, Ts, 16 * mt, Vc, x_c0);
        }
        __syncthreads();

        // (e) Z = U - W S ; O = Q S
        warp_gemm<DK, NT_X, DK, false, NX, true>(z, Ws, 16 * mt, Xb, x_c0);
        float o[NT_X][4];
        if constexpr (HAS_Q) {
            zero_frag(o);
            warp_gemm<DK, NT_X, DK, false, NX, true>(o, Qc, 16 * mt, Xb, x_c0);
            if constexpr (GATED) {
                // readout of the decayed state: row l of Q S times lambda[1:l]
#pragma unroll
                for (int nt = 0; nt < NT_X; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[nt][e] *= lam_l[16 * mt + g8 + 8 * (e >> 1)];
            }
        }
        store_frag<NT_X, NX>(Zs, 16 * mt, x_c0, z, 1.f);
        if constexpr (GATED) {
            // K's other uses are done: scale its rows by lambda[l+1:C] for the state
            // update, and decay the state by lambda[1:C]
            constexpr int V = 16 / sizeof(E);
            E* Kw = const_cast<E*>(Kc);
            for (int idx = tid; idx < kChunk * (DK / V); idx += kThreads) {
                const float f = lam_r[idx / (DK / V)];
                E* c = Kw + idx * V;  // swizzling permutes chunks within a row only
#pragma unroll
                for (int j = 0; j < V; ++j) c[j] = to_e<E>(float(c[j]) * f);
            }
            const float fc = lam_c[0];
#pragma unroll
            for (int m = 0; m < MT_S; ++m)
#pragma unroll
                for (int nt = 0; nt < NT_X; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) s[m][nt][e] *= fc;
        }
        if constexpr (KDA) {
            // the state's key rows decay by lambda[1:C] of their channel
#pragma unroll
            for (int m = 0; m < MT_S; ++m)
#pragma unroll
                for (int nt = 0; nt < NT_X; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) s[m][nt][e] *= lamc_k[s_r0 + 16 * m + g8 + 8 * (e >> 1)];
        }
        __syncthreads();

        // (f) O += (Q K^T o M_c) Z
        if constexpr (HAS_Q) {
            warp_gemm<kChunk, NT_X, kChunk, false, NX, true>(o, Ps, 16 * mt, Zs, x_c0);
            store_frag<NT_X, NX>(Os, 16 * mt, x_c0, o, 1.f);
        }
        // (g) S += K^T Z
#pragma unroll
        for (int m = 0; m < MT_S; ++m)
            warp_gemm<kChunk, NT_X, DK, true, NX, true>(s[m], Kc, s_r0 + 16 * m, Zs, x_c0);
        __syncthreads();

        // (h) O tile -> global
        if (HAS_Q) {
            constexpr int V = 16 / sizeof(E);
            constexpr int CPR = NX / V;
            const int t0 = it.tok0 + r * kChunk;
            const int rows = min(kChunk, it.tok1 - t0);
            for (int idx = tid; idx < kChunk * CPR; idx += kThreads) {
                const int rr = idx / CPR, c = idx % CPR;
                const int m = t0 + rr;
                // one output row per token: the last of its nsub steps
                if (rr < rows && m % nsub == nsub - 1)
                    *reinterpret_cast<int4*>(og + (int64_t)(m / nsub) * p.o_st + c * V) =
                        *reinterpret_cast<const int4*>(Os + SW::template off<NX>(rr, c * V));
            }
        }
    }

    if (x_out) {
#pragma unroll
        for (int m = 0; m < MT_S; ++m)
#pragma unroll
            for (int nt = 0; nt < NT_X; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int r = s_r0 + 16 * m + g8 + 8 * h;
                    const int c = x_c0 + 8 * nt + 2 * t4;
                    *reinterpret_cast<float2*>(x_out + r * NX + c) =
                        make_float2(s[m][nt][2 * h], s[m][nt][2 * h + 1]);
                }
    }
}

template <typename E, int DK, int DV, int STAGES, bool GATED, bool KDA = false>
__global__ void __launch_bounds__(kThreads, 1) k_boundary(Params p) {
    extern __shared__ __align__(128) char smem[];
    const int n = count_C(p.sched);
    for (int i = blockIdx.x; i < n; i += gridDim.x) {
        const Item it = item_C(p.sched, i);
        run_segment<E, DK, DV, true, true, STAGES, GATED, KDA>(p, it, kModeOut, smem);
        __syncthreads();
    }
}

template <typename E, int DK, int DV, int STAGES, bool GATED, bool KDA = false>
__global__ void __launch_bounds__(kThreads, 1) k_summary(Params p) {
    extern __shared__ __align__(128) char smem[];
    const int n = count_A(p.sched);
    for (int i = blockIdx.x; i < n; i += gridDim.x) {
        int mode;
        const Item it = item_A(p.sched, i, mode);
        if (mode == kModeHP) {
            // both maps of the segment, one after the other
            run_segment<E, DK, DV, true, false, STAGES, GATED, KDA>(p, it, kModeH, smem);
            __syncthreads();
            run_segment<E, DK, DK, false, false, STAGES, GATED, KDA>(p, it, kModeP, smem);
        } else if (mode == kModeP) {
            run_segment<E, DK, DK, false, false, STAGES, GATED, KDA>(p, it, mode, smem);
        } else {
            run_segment<E, DK, DV, true, false, STAGES, GATED, KDA>(p, it, mode, smem);
        }
        __syncthreads();
    }
}

// Segment scan: start(g+1) = P_g start(g) + H_g, start(1) = end state of
// segment 0.  One CTA per (chain, COLS columns of the state); warp w computes
// state rows 16 w .. + 15 of the CTA's columns with tensor-core tf32 products
// in three passes (hi hi + hi lo + lo hi, the operands split into a tf32 head
// and a tf32 tail), which keeps the sums at fp32 accuracy.  P_{g+1} is
// prefetched by TMA (boxes of 32 columns, 128-byte swizzle, so that the
// fragment reads of 8 rows hit distinct banks) and each thread's H_{g+1}
// values into registers while step g is computed; the CTA's state columns are
// kept transposed with rows padded by 4 floats.  COLS is 16 when 8-column CTAs
// would need more than one wave.
template <int DK, int COLS>
__host__ __device__ constexpr int scan_threads() { return 2 * DK; }
template <int DK, int COLS>
__host__ __device__ constexpr int scan_smem_bytes() {
    return 2 * DK * DK * 4 + COLS * (DK + 4) * 4 + 32 + 1024;
}
#ifdef DN_TRACE
static __device__ unsigned long long g_dn_trace_scan[64 * 4];
#define DN_TSC(g, slot)                                                                   \
    do {                                                                                  \
        if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && (g) < 64)            \
            g_dn_trace_scan[(g) * 4 + (slot)] = sm100::globaltimer();                     \
    } while (0)
#else
#define DN_TSC(g, slot) \
    do {                \
    } while (0)
#endif
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = sm100::to_tf32(x);
    lo = sm100::to_tf32(x - __uint_as_float(hi));
}
template <int DK, int DV, int COLS>
__global__ void __launch_bounds__(2 * DK) k_scan(const __grid_constant__ CUtensorMap tp, Params p) {
    extern __shared__ uint8_t scan_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(scan_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    constexpr int SLD = DK + 4;                 // padded row of a transposed state column
    constexpr int NTILE = COLS / 8;             // n8 tiles
    constexpr uint32_t kPBytes = (uint32_t)DK * DK * 4u;
    static_assert(DK % 32 == 0 && COLS % 8 == 0, "tiles");
    auto Pm = [&](int b) { return smem + b * kPBytes; };    // DK/32 swizzled boxes of DK rows x 32 columns
    float* St = reinterpret_cast<float*>(smem + 2 * kPBytes);  // COLS x SLD
    uint64_t* bars = reinterpret_cast<uint64_t*>(St + COLS * SLD);
    sm100::WaitCtl* ctl = reinterpret_cast<sm100::WaitCtl*>(bars + 2);
    volatile int* abort_flag = &ctl->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
    const int ra = 16 * warp + gq;              // fragment rows ra, ra + 8
    const int c0 = blockIdx.y * COLS;
    const int n = count_scan(p.sched);
    if (tid == 0) {
        sm100::mbar_init(&bars[0], 1);
        sm100::mbar_init(&bars[1], 1);
        sm100::wait_ctl_init(ctl, p.wait_ns);
        sm100::mbar_fence_init();
    }
    __syncthreads();
    // per buffer (bit b): parity of its next completion, and a copy in flight into
    // it (at most one: a buffer is refilled only after its last step was computed)
    uint32_t phase = 0, pending = 0;
    float2 hn[NTILE][2];
    // P_g into buffer g % 2, this thread's fragment of H_g into hn
    auto prefetch = [&](const Item& it, int g) {
        if (g + 1 >= it.G) return;
        const int b = g & 1;
        pending |= 1u << b;
        if (tid == 0) {
            sm100::mbar_expect_tx(&bars[b], kPBytes);
#pragma unroll
            for (int bx = 0; bx < DK / 32; ++bx)
                sm100::tma_load_2d(Pm(b) + bx * DK * 128, &tp, &bars[b], 32 * bx, (it.slot + g) * DK);
        }
        const float* Hg = p.wsH + (int64_t)(it.slot + g) * DK * DV + c0 + 2 * tq;
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                hn[nt][h] = *reinterpret_cast<const float2*>(Hg + (int64_t)(ra + 8 * h) * DV + 8 * nt);
    };
    // element (r, k) of a P buffer
    auto pel = [&](const uint8_t* pb, int r, int k) {
        return *reinterpret_cast<const float*>(pb + (k >> 5) * (DK * 128) + r * 128 +
                                               ((((k & 31) >> 2) ^ (r & 7)) << 4) + ((k & 3) << 2));
    };
    bool ok = true;
    for (int i = blockIdx.x; ok && i < n; i += gridDim.x) {
        const Item it = item_scan(p.sched, i);
        const float* E0 = p.wsH + (int64_t)it.slot * DK * DV;
        float* out0 = p.wsS + (int64_t)it.slot * DK * DV;
        prefetch(it, 1);
        for (int e = tid; e < DK * COLS; e += 2 * DK) {
            const int r = e % DK, cc = e / DK;
            const float x = E0[r * DV + c0 + cc];
            St[cc * SLD + r] = x;
            out0[r * DV + c0 + cc] = x;
        }
        DN_TSC(0, 0);
        for (int g = 1; g + 1 < it.G; ++g) {
            DN_TSC(g, 0);
            // four independent accumulations (even / odd k steps, head x head / the
            // two head x tail terms) keep several products in flight per warp
            float acc[NTILE][4], accH[NTILE][4], accL[2][NTILE][4];
#pragma unroll
            for (int nt = 0; nt < NTILE; ++nt) {
                acc[nt][0] = hn[nt][0].x; acc[nt][1] = hn[nt][0].y;
                acc[nt][2] = hn[nt][1].x; acc[nt][3] = hn[nt][1].y;
#pragma unroll
                for (int e = 0; e < 4; ++e) accH[nt][e] = accL[0][nt][e] = accL[1][nt][e] = 0.f;
            }
            prefetch(it, g + 1);
            const int b = g & 1;
            const bool landed = sm100::mbar_wait(&bars[b], (phase >> b) & 1u, abort_flag);
            if (landed) {
                phase ^= 1u << b;
                pending &= ~(1u << b);
            }
            if (__syncthreads_or(!landed)) {  // also: S(g) is written
                ok = false;
                break;
            }
            DN_TSC(g, 1);
            const uint8_t* pb = Pm(b);
#pragma unroll
            for (int ks = 0; ks < DK / 8; ++ks) {
                const int k = 8 * ks + tq;
                uint32_t ah[4], al[4];
                split_tf32(pel(pb, ra, k), ah[0], al[0]);
                split_tf32(pel(pb, ra + 8, k), ah[1], al[1]);
                split_tf32(pel(pb, ra, k + 4), ah[2], al[2]);
                split_tf32(pel(pb, ra + 8, k + 4), ah[3], al[3]);
#pragma unroll
                for (int nt = 0; nt < NTILE; ++nt) {
                    const float* sc = St + (8 * nt + gq) * SLD + k;
                    uint32_t bh0, bl0, bh1, bl1;
                    split_tf32(sc[0], bh0, bl0);
                    split_tf32(sc[4], bh1, bl1);
                    float (&hacc)[4] = (ks & 1) ? accH[nt] : acc[nt];
                    sm100::mma_tf32(accL[ks & 1][nt], al[0], al[1], al[2], al[3], bh0, bh1);
                    sm100::mma_tf32(accL[ks & 1][nt], ah[0], ah[1], ah[2], ah[3], bl0, bl1);
                    sm100::mma_tf32(hacc, ah[0], ah[1], ah[2], ah[3], bh0, bh1);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[nt][e] += accH[nt][e] + (accL[0][nt][e] + accL[1][nt][e]);
            __syncthreads();  // every thread has read S(g) and P_g
            DN_TSC(g, 2);
            float* outg = p.wsS + (int64_t)(it.slot + g) * DK * DV + c0 + 2 * tq;
#pragma unroll
            for (int nt = 0; nt < NTILE; ++nt) {
                const int cc = 8 * nt + 2 * tq;
                St[cc * SLD + ra] = acc[nt][0];
                St[(cc + 1) * SLD + ra] = acc[nt][1];
                St[cc * SLD + ra + 8] = acc[nt][2];
                St[(cc + 1) * SLD + ra + 8] = acc[nt][3];
                *reinterpret_cast<float2*>(outg + (int64_t)ra * DV + 8 * nt) = make_float2(acc[nt][0], acc[nt][1]);
                *reinterpret_cast<float2*>(outg + (int64_t)(ra + 8) * DV + 8 * nt) = make_float2(acc[nt][2], acc[nt][3]);
            }
        }
        __syncthreads();
    }
    // copies still in flight must land before the CTA exits (also after a time-out)
    if (tid == 0) {
        volatile int drain = 0;
        for (int b = 0; b < 2; ++b)
            if ((pending >> b) & 1u) sm100::mbar_wait(&bars[b], (phase >> b) & 1u, &drain, sm100::kDrainWaitNs);
        if (*abort_flag) atomicExch(p.err, kErrTimeout);
    }
}

}  // namespace dn
