// Kimi Delta Attention: the chunk-parallel pre-pass of the tensor-core path
// (bf16, d_k = d_v = 128).
//
// "Linear Attention, Visualized", section "Kimi Delta Attention (KDA)", complete
// per-chunk algorithm: every key channel c decays by its own a_t[c] = exp(g_t[c]).
// With G_l = g_1 + ... + g_l per channel (within the chunk) the chunk's factors are
//   L[l][m] = sum_c k_l[c] k_m[c] exp(G_l[c] - G_m[c])   (m < l)
//   P[l][m] = sum_c q_l[c] k_m[c] exp(G_l[c] - G_m[c])   (m <= l)
//   T = (I + B L)^{-1} B,  Q<- = exp(G) o Q,  K<- = exp(G) o K,  K-> = exp(G_C - G) o K,
//   lambda[1:C] = exp(G_C) per channel.
// The chain kernels then need no gate arithmetic: W = T K<-, U = T V,
// Z = U - W S, O = Q<- S + P Z, S' = Diag(lambda[1:C]) S + K->^T Z.
// Like "Context Parallelism for DeltaNet", section 2, step 1, all of it depends only on
// the chunk's own inputs, so one CTA forms one (chunk, head) unit at a time and the
// units run in parallel.  L and P are formed block by block of 16 rows against the
// block's first row s (exp(G_l - G_m) = exp(G_l - G_s) exp(G_s - G_m)), which keeps
// every factor in range for |g| < 5.8 per token and channel (see dn_chain.cuh).
//
// Per unit a CTA (8 warps, two per SM) waits for the chunk's k, q, beta and log decays
// (copies issued while the previous unit's solve ran), forms the running sums, loads each
// thread's four rows of running sums and k (piece c8 = tid % 16 of rows tid / 16 + 16 i)
// into registers, builds the four Gram blocks (operand rows scaled 8 channels at a time,
// one fast exponential per element, then mma.sync warp products), stores Q<-, K<- and K->
// straight from registers into the unit, solves for T and copies T and P out.
//
// Unit layout in the workspace (66,560 bytes per (chunk, head)): T and P (bf16 64 x 64,
// 128-byte rows, 16-byte pieces swizzled by row % 8: the tensor cores' operand layout),
// Q<-, K<-, K-> (each two boxes of 64 channels x 64 rows in the same layout, the layout a
// TMA load of the tile would give), lambda[1:C] per channel (fp32).
#pragma once

#include "dn_chain.cuh"
#include "dn_common.cuh"
#include "dn_warp_gemm.cuh"

namespace dn {

#ifdef DN_TRACE
static __device__ unsigned long long g_dn_trace_kda[16 * 8];
#define DN_TRK(k, slot)                                                               \
    do {                                                                              \
        if (blockIdx.x == 0 && (k) < 16 && threadIdx.x == 0) {                         \
            unsigned long long t_;                                                    \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                    \
            g_dn_trace_kda[(k) * 8 + (slot)] = t_;                                    \
        }                                                                             \
    } while (0)
#else
#define DN_TRK(k, slot) \
    do {                \
    } while (0)
#endif

constexpr int kKdaUnitT = 0, kKdaUnitP = 8192, kKdaUnitQL = 16384, kKdaUnitKL = 32768, kKdaUnitKR = 49152,
              kKdaUnitF = 65536, kKdaUnitFBytes = 512;
constexpr int kKdaUnitBytes = 66560;

// Shared memory of the KDA pre-pass (byte offsets).  [0, OFF_AF) holds the chunk's k, q,
// log decays and the block operands until the scaled tiles are written out.  The solve
// then keeps N where the right operand was and writes T over A, so that the next unit's
// k, q, log decays and beta load into [0, OFF_R) and OFF_BNEXT while it runs.
struct KdaPrepLay {
    static constexpr int DK = 128;
    static constexpr int OFF_K = 0;          // 64 x 128 bf16 (Swz): K
    static constexpr int OFF_Q = 16384;      // 64 x 128 bf16 (Swz): Q
    static constexpr int OFF_G = 32768;      // 64 x 128 fp32: log decays, later running sums
    static constexpr int OFF_R = 65536;      // 64 x 128 bf16 (Swz): a block's right operand
    static constexpr int OFF_LQ = 81920;     // 32 x 128 bf16 (Swz): a block's left operands [K; Q]
    static constexpr int OFF_N = 65536;      // after the tiles: N, 64 x 65 fp32
    static constexpr int OFF_X = 82176;      //   the fp32 solve's staging (the bf16 solve stages in N)
    static constexpr int OFF_BNEXT = 89856;  //   the next unit's beta, 64 fp32
    static constexpr int OFF_AF = 90112;     // A = B L, 64 x 65 fp32; T (64 x 64 bf16, Swz) once the solve has read A
    static constexpr int OFF_T = OFF_AF;
    static constexpr int OFF_P = 106752;     // P, 64 x 64 bf16 (Swz)
    static constexpr int OFF_BETA = 114944;  // 64 fp32
    static constexpr int OFF_LAMC = 115200;  // lambda[1:C], 128 fp32
    static constexpr int TOTAL = 115712;     // two CTAs per SM
};
static_assert(KdaPrepLay::OFF_N + 64 * 65 * 4 <= KdaPrepLay::OFF_X && KdaPrepLay::OFF_X + 3 * 256 * 4 <= KdaPrepLay::OFF_BNEXT &&
                  KdaPrepLay::OFF_BNEXT + 64 * 4 <= KdaPrepLay::OFF_AF && KdaPrepLay::OFF_R == KdaPrepLay::OFF_N,
              "the solve's tiles stay clear of the next unit's loads");

// bf16 pair (lo, hi) times (fa, fb), rounded to nearest-even.
__device__ __forceinline__ uint32_t kda_scale2(uint32_t w, float fa, float fb) {
    return sm100::pack_bf16(__uint_as_float(w << 16) * fa, __uint_as_float(w & 0xffff0000u) * fb);
}
__device__ __forceinline__ uint4 kda_scale8(uint4 v, const float (&f)[8]) {
    return make_uint4(kda_scale2(v.x, f[0], f[1]), kda_scale2(v.y, f[2], f[3]), kda_scale2(v.z, f[4], f[5]),
                      kda_scale2(v.w, f[6], f[7]));
}
// the 8 running sums of row r, channels 8 c8 .. 8 c8 + 7.  Pieces c8 with bit 2 set read their
// second half first: a quarter warp's 16-byte reads (pieces 32 bytes apart) then fall in eight
// distinct groups of four banks.
__device__ __forceinline__ void kda_row8(const float* G, int r, int c8, float (&g)[8]) {
    const int sw = (c8 >> 2) & 1;
    const float4* src = reinterpret_cast<const float4*>(G + r * KdaPrepLay::DK + 8 * c8);
    const float4 x = src[sw];
    const float4 y = src[sw ^ 1];
    const float4 a = sw ? y : x, b = sw ? x : y;
    g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w; g[4] = b.x; g[5] = b.y; g[6] = b.z; g[7] = b.w;
}

template <int DK>
static __global__ void __launch_bounds__(kThreads, 2) k_kda_prep(Params p) {
    static_assert(DK == KdaPrepLay::DK, "the tensor-core path has d_k = 128");
    using E = __nv_bfloat16;
    using SW = Swz<E>;
    using L = KdaPrepLay;
    constexpr int LD = 65;  // fp32 solve tiles
    extern __shared__ __align__(128) char kda_smem[];
    E* Kc = reinterpret_cast<E*>(kda_smem + L::OFF_K);
    E* Qc = reinterpret_cast<E*>(kda_smem + L::OFF_Q);
    float* G = reinterpret_cast<float*>(kda_smem + L::OFF_G);
    E* Rs = reinterpret_cast<E*>(kda_smem + L::OFF_R);
    E* LQs = reinterpret_cast<E*>(kda_smem + L::OFF_LQ);
    float* Nf = reinterpret_cast<float*>(kda_smem + L::OFF_N);
    float* Xt = reinterpret_cast<float*>(kda_smem + L::OFF_X);
    E* Ts = reinterpret_cast<E*>(kda_smem + L::OFF_T);
    float* Af = reinterpret_cast<float*>(kda_smem + L::OFF_AF);
    E* Ps = reinterpret_cast<E*>(kda_smem + L::OFF_P);
    float* bc = reinterpret_cast<float*>(kda_smem + L::OFF_BETA);
    float* lamc = reinterpret_cast<float*>(kda_smem + L::OFF_LAMC);
    float* bnext = reinterpret_cast<float*>(kda_smem + L::OFF_BNEXT);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    const int H = p.sched.H;
    const int units = count_chunks(p.sched) * H;
    // the scaled-operand passes work on 16-byte pieces of 8 channels: thread tid always
    // takes piece c8 of rows tid / 16, tid / 16 + 16, ... (a Swz tile row r keeps piece c8
    // at byte r * 256 + ((c8 ^ (r % 8)) * 16))
    const int c8 = tid & 15, r16 = tid >> 4;
    auto piece = [](int r, int c) { return r * 256 + ((c ^ (r & 7)) << 4); };
    uint8_t* Kb = reinterpret_cast<uint8_t*>(Kc);
    uint8_t* Qb = reinterpret_cast<uint8_t*>(Qc);
    uint8_t* Rb = reinterpret_cast<uint8_t*>(Rs);
    uint8_t* LQb = reinterpret_cast<uint8_t*>(LQs);

    // unit uu's k, q, beta and log decays (rows past the chunk: zeros, identity steps), as
    // one group of asynchronous copies
    auto issue_loads = [&](int uu) {
        const int head = uu % H;
        int b, t0, t1;
        chunk_range(p.sched, uu / H, b, t0, t1);
        const int rows = t1 - t0;
        const E* kg = static_cast<const E*>(p.k) + b * p.k_sb + head * p.k_sh;
        const E* qg = static_cast<const E*>(p.q) + b * p.q_sb + head * p.q_sh;
        const float* bg = p.beta + b * p.b_sb + head * p.b_sh;
        const float* gg = p.g + b * p.g_sb + head * p.g_sh;
        load_tile<E, DK>(Kc, kg + (int64_t)t0 * p.k_st, p.k_st, rows);
        load_tile<E, DK>(Qc, qg + (int64_t)t0 * p.q_st, p.q_st, rows);
        if (tid < kChunk) {
            const bool ok = tid < rows;
            cp_async4(smem_addr(bnext + tid), ok ? bg + (int64_t)(t0 + tid) * p.b_st : bg, ok ? 4 : 0);
        }
        for (int idx = tid; idx < kChunk * (DK / 4); idx += kThreads) {
            const int rr = idx / (DK / 4), c = idx % (DK / 4);
            const bool ok = rr < rows;
            const float* src = ok ? gg + (int64_t)(t0 + rr) * p.g_st + 4 * c : gg;
            cp_async16(smem_addr(G + rr * DK + 4 * c), src, ok ? 16 : 0);
        }
        cp_async_commit();
    };

    if (blockIdx.x < units) issue_loads(blockIdx.x);
    int it_ = 0;
#pragma unroll 1
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++it_) {
        DN_TRK(it_, 0);
        uint8_t* unit = p.wsT + (size_t)u * kKdaUnitBytes;
        cp_async_wait<0>();
        __syncthreads();
        DN_TRK(it_, 1);
        if (tid < kChunk) bc[tid] = bnext[tid];  // before the block operands take OFF_BNEXT

        // running sums per key channel, in place, and lambda[1:C]
        if (tid < DK) {
            float acc = 0.f;
            for (int l = 0; l < kChunk; ++l) {
                acc += G[l * DK + tid];
                G[l * DK + tid] = acc;
            }
            lamc[tid] = expf(acc);
        }
        __syncthreads();
        DN_TRK(it_, 2);

        // the thread's rows r16 + 16 i (i = 0..3), piece c8: running sums and k, held in
        // registers through the Gram blocks and the decayed tiles
        float gr[4][8];
        uint4 kr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            kda_row8(G, r16 + 16 * i, c8, gr[i]);
            kr[i] = *reinterpret_cast<const uint4*>(Kb + piece(r16 + 16 * i, c8));
        }

        // rows 16 b .. 16 b + 15 of A = B L (fp32, strict lower) and of P (inclusive),
        // against reference row s = 16 b
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            const int s = 16 * blk, ncol = s + 16;
            float gs[8];
            kda_row8(G, s, c8, gs);
            // right operand rows m = r16 + 16 i < ncol: k_m o exp(G_s - G_m)
#pragma unroll
            for (int i = 0; i <= blk; ++i) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __expf(gs[e] - gr[i][e]);
                *reinterpret_cast<uint4*>(Rb + piece(r16 + 16 * i, c8)) = kda_scale8(kr[i], f);
            }
            // left operands, rows l = s + r16 of the block: k_l and q_l o exp(G_l - G_s)
            {
                const int l = s + r16;
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __expf(gr[blk][e] - gs[e]);
                *reinterpret_cast<uint4*>(LQb + piece(r16, c8)) = kda_scale8(kr[blk], f);
                *reinterpret_cast<uint4*>(LQb + piece(16 + r16, c8)) =
                    kda_scale8(*reinterpret_cast<const uint4*>(Qb + piece(l, c8)), f);
            }
            // the block's rows right of its last column are zero in both
            for (int idx = tid; idx < 16 * (kChunk - ncol); idx += kThreads) {
                const int row = s + idx / (kChunk - ncol), col = ncol + idx % (kChunk - ncol);
                Af[row * LD + col] = 0.f;
                Ps[SW::template off<kChunk>(row, col)] = __float2bfloat16_rn(0.f);
            }
            __syncthreads();
            const int ntile = blk + 1;
            if (warp < 2 * ntile) {
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
                        if (mat == 0) Af[row * LD + col] = col < row ? bc[row] * acc[nt][e] : 0.f;
                        else acc[nt][e] = col > row ? 0.f : acc[nt][e];
                    }
                if (mat == 1) store_frag<2, kChunk>(Ps, s, 16 * j, acc, 1.f);
            }
            __syncthreads();
        }

        DN_TRK(it_, 3);
        // K<- = exp(G) o K, K-> = exp(G_C - G) o K, Q<- = exp(G) o Q, stored straight to the
        // unit's boxes: logical piece c8 of row l sits in box c8 / 8 at row l, piece
        // (c8 % 8) ^ (l % 8) (a warp writes whole 128-byte box rows)
        {
            float gC[8];
            kda_row8(G, kChunk - 1, c8, gC);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int l = r16 + 16 * i;
                float fl[8], fr[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    fl[e] = __expf(gr[i][e]);
                    fr[e] = __expf(gC[e] - gr[i][e]);
                }
                const int go = (c8 >> 3) * 8192 + l * 128 + (((c8 & 7) ^ (l & 7)) << 4);
                *reinterpret_cast<uint4*>(unit + kKdaUnitKL + go) = kda_scale8(kr[i], fl);
                *reinterpret_cast<uint4*>(unit + kKdaUnitKR + go) = kda_scale8(kr[i], fr);
                *reinterpret_cast<uint4*>(unit + kKdaUnitQL + go) =
                    kda_scale8(*reinterpret_cast<const uint4*>(Qb + piece(l, c8)), fl);
            }
        }
        if (tid < DK / 4)
            reinterpret_cast<float4*>(unit + kKdaUnitF)[tid] = reinterpret_cast<const float4*>(lamc)[tid];
        __syncthreads();  // k, q, the log decays and the right operand are read
        DN_TRK(it_, 4);
        if (u + (int)gridDim.x < units) issue_loads(u + gridDim.x);

        // T = (I + B L)^{-1} B
        ut_solve<E>(Af, Nf, Xt, bc, Ts);
        __syncthreads();
        DN_TRK(it_, 5);
        for (int idx = tid; idx < 2 * 512; idx += kThreads) {
            const int t = idx >> 9, pc = idx & 511;
            const uint8_t* src = reinterpret_cast<const uint8_t*>(t == 0 ? Ts : Ps);
            *reinterpret_cast<uint4*>(unit + (t == 0 ? kKdaUnitT : kKdaUnitP) + pc * 16) =
                *reinterpret_cast<const uint4*>(src + pc * 16);
        }
        __syncthreads();  // the next unit's block operands overwrite the tiles
        DN_TRK(it_, 6);
    }
}

}  // namespace dn
