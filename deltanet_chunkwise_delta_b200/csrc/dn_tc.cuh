// Tensor-core (tcgen05 / TMEM / TMA) chain kernel for bf16, d_k = d_v = 128.
//
// Same per-chunk algorithm as dn_chain.cuh ("Linear Attention, Visualized",
// DeltaNet, "Complete per-chunk algorithm"), evaluated in the transposed
// domain so that every tensor-core product has M = 128:
//   G   = [Q; K] K^T                      (rows: 64 queries, then 64 keys)
//   A   = B L from the key rows of G;  P = (Q K^T) o M_c from the query rows
//   T   = (I + B L)^{-1} B               (blocked solve: fp32 diagonal blocks,
//                                          tf32 mma.sync off-diagonal blocks)
//   W^T = K^T T^T,  U^T = V^T T^T
//   Z^T = U^T - S^T W^T                  (accumulated into U^T's columns)
//   O^T = S^T Q^T + Z^T P^T
//   S^T <- S^T + Z^T K
// S^T (d_v lanes x d_k columns, fp32) lives in tensor memory for the whole run;
// a bf16 copy in shared memory feeds the next chunk's products.
//
// Warp roles (448 threads):
//   warps 0-7   chain epilogue: Z^T -> bf16, S^T -> bf16, O -> global
//   warps 8-11  chunk-parallel epilogue: G -> A, P; solve -> T; W^T -> W
//   warp 12     issues every tcgen05.mma (one thread)
//   warp 13     issues the TMA loads of q, k, v (one thread)
// The chunk-parallel work of chunk r+1 overlaps the state chain of chunk r.
// Every wait on an mbarrier is bounded; on time-out the CTA drains, frees
// its tensor memory and reports DN_ERR_TIMEOUT through the error flag.
#pragma once

#include "dn_common.cuh"
#include "dn_sm100.cuh"

namespace dn {
namespace tc {

using namespace sm100;

constexpr int D = 128;
constexpr int kThreadsTc = 448;
constexpr int kMmaWarp = 12;
constexpr int kTmaWarp = 13;

// shared memory (byte offsets from a 1024-aligned base)
constexpr int STAGE_BYTES = 49152;  // [Q|K] for d 0-63, [Q|K] for d 64-127, V (2 x 8 KB)
constexpr int OFF_WB = 2 * STAGE_BYTES;
constexpr int OFF_TB = OFF_WB + 16384;
constexpr int OFF_PB = OFF_TB + 2 * 8192;
constexpr int OFF_ZB = OFF_PB + 2 * 8192;
constexpr int OFF_SBF = OFF_ZB + 16384;
constexpr int BLK_LD = 17;
constexpr int BLK_FLOATS = 16 * BLK_LD;
constexpr int OFF_ABLK = OFF_SBF + 32768;
constexpr int OFF_NBLK = OFF_ABLK + 10 * BLK_FLOATS * 4;
constexpr int OFF_XS = OFF_NBLK + 10 * BLK_FLOATS * 4;
constexpr int OFF_BETA = OFF_XS + 4 * BLK_FLOATS * 4;
constexpr int OFF_BAR = OFF_BETA + 2 * 64 * 4;
constexpr int NBAR = 16;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM_USED = OFF_MISC + 64;
constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment

// tensor-memory columns (512 allocated)
constexpr uint32_t TM_S = 0, TM_O = 128, TM_ZU = 192, TM_WT = 320, TM_G = 384;

enum : int {
    B_FULL = 0,   // +stage: TMA landed
    B_EMPTY = 2,  // +stage: stage consumed by the MMAs
    B_GFULL = 4,  // G ready in TMEM
    B_GFREE,      // G read by the solve warps
    B_TFULL,      // T, P written to shared memory
    B_WUFULL,     // W^T, U^T ready in TMEM
    B_WFULL,      // W written to shared memory
    B_C1A,        // Z^T = U^T - S^T W^T complete
    B_ZFULL,      // Z^T (bf16) written
    B_SFULL,      // S^T updated
    B_OFULL,      // O^T complete
    B_SBF,        // bf16 copy of S^T written
    B_OFREE,      // O^T read out
};

__device__ __forceinline__ int bidx(int bi, int bj) { return bi * (bi + 1) / 2 + bj; }

// acc (16 x 16, two n8 tiles) += A (16 x 16) * B (16 x 16); fp32 tiles, row stride 17.
__device__ __forceinline__ void mm16(float (&acc)[2][4], const float* A, const float* B) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a0 = to_tf32(A[g * BLK_LD + 8 * ks + t]);
        const uint32_t a1 = to_tf32(A[(g + 8) * BLK_LD + 8 * ks + t]);
        const uint32_t a2 = to_tf32(A[g * BLK_LD + 8 * ks + t + 4]);
        const uint32_t a3 = to_tf32(A[(g + 8) * BLK_LD + 8 * ks + t + 4]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b0 = to_tf32(B[(8 * ks + t) * BLK_LD + 8 * nt + g]);
            const uint32_t b1 = to_tf32(B[(8 * ks + t + 4) * BLK_LD + 8 * nt + g]);
            mma_tf32(acc[nt], a0, a1, a2, a3, b0, b1);
        }
    }
}

__device__ __forceinline__ void st16(float* C, const float (&acc)[2][4], float scale) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        C[g * BLK_LD + 8 * nt + 2 * t] = scale * acc[nt][0];
        C[g * BLK_LD + 8 * nt + 2 * t + 1] = scale * acc[nt][1];
        C[(g + 8) * BLK_LD + 8 * nt + 2 * t] = scale * acc[nt][2];
        C[(g + 8) * BLK_LD + 8 * nt + 2 * t + 1] = scale * acc[nt][3];
    }
}

// 32 fp32 values -> 4 swizzled 16-byte chunks (bf16) of row r, columns c0..c0+31.
__device__ __forceinline__ void st_row32_bf16(uint8_t* tile, int r, int c0, const uint32_t (&v)[32]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
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
    float* betas = reinterpret_cast<float*>(smem + OFF_BETA);
    float* Ablk = reinterpret_cast<float*>(smem + OFF_ABLK);
    float* Nblk = reinterpret_cast<float*>(smem + OFF_NBLK);
    float* Xs = reinterpret_cast<float*>(smem + OFF_XS);
    uint8_t* Wb = smem + OFF_WB;
    uint8_t* Zb = smem + OFF_ZB;
    uint8_t* Sbf = smem + OFF_SBF;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bars[B_FULL + 0], 1);
        mbar_init(&bars[B_FULL + 1], 1);
        mbar_init(&bars[B_EMPTY + 0], 1);
        mbar_init(&bars[B_EMPTY + 1], 1);
        mbar_init(&bars[B_GFULL], 1);
        mbar_init(&bars[B_GFREE], 128);
        mbar_init(&bars[B_TFULL], 128);
        mbar_init(&bars[B_WUFULL], 1);
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
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (!HAS_Q && warp < 8) {
        // the query rows of G are not used without output; keep them finite
        for (int i = threadIdx.x; i < 4 * 8192 / 16; i += 256) {
            const int part = i / 512, off = (i % 512) * 16;   // part: stage * 2 + atom
            *reinterpret_cast<uint4*>(smem + (part >> 1) * STAGE_BYTES + (part & 1) * 16384 + off) =
                make_uint4(0, 0, 0, 0);
        }
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
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && nch > 0) {
            const uint32_t bytes = (HAS_Q ? 16384u : 0u) + 16384u + (has_v ? 16384u : 0u);
            int issued = 0;
            for (int r = 0; r < nch; ++r) {
                const int s = r & 1;
                if (r >= 2 && !mbar_wait(&bars[B_EMPTY + s], ((r >> 1) - 1) & 1, abort_flag)) break;
                mbar_expect_tx(&bars[B_FULL + s], bytes);
                uint8_t* st = smem + s * STAGE_BYTES;
                const int t0 = it.tok0 + r * kChunk;
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    if (HAS_Q) tma_load_4d(st + a * 16384, &tq, &bars[B_FULL + s], a * 64, it.head, t0, it.b);
                    tma_load_4d(st + a * 16384 + 8192, &tk, &bars[B_FULL + s], a * 64, it.head, t0, it.b);
                    if (has_v)
                        tma_load_4d(st + 32768 + a * 8192, &tv, &bars[B_FULL + s], a * 64, it.head, t0, it.b);
                }
                issued = r + 1;
            }
            // the last loads issued must have landed before the CTA may exit
            for (int r = issued - 2 < 0 ? 0 : issued - 2; r < issued; ++r)
                mbar_wait(&bars[B_FULL + (r & 1)], (r >> 1) & 1, abort_flag, 200000000ull);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && nch > 0) {
            const uint32_t sb = saddr(smem);
            const uint32_t i_g = idesc_bf16(128, 64, false, false);
            const uint32_t i_tt = idesc_bf16(128, 64, true, false);
            const uint32_t i_c1a = idesc_bf16(128, 64, false, false, true);
            const uint32_t i_c1b = idesc_bf16(128, 64, false, false);
            const uint32_t i_c3 = idesc_bf16(128, 128, false, true);
            const uint32_t i_c2 = idesc_bf16(128, 64, false, false);
            bool ok = true;
            auto m1 = [&](int r) -> bool {
                const int s = r & 1;
                if (!mbar_wait(&bars[B_FULL + s], (r >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t st = sb + s * STAGE_BYTES;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t rg = st + (j >> 2) * 16384 + (j & 3) * 32;
                    umma_bf16(tmem + TM_G, sdesc(rg, 16, 1024), sdesc(rg + 8192, 16, 1024), i_g, j > 0);
                }
                umma_commit(&bars[B_GFULL]);
                return true;
            };
            auto m23 = [&](int r) -> bool {
                const int s = r & 1;
                if (!mbar_wait(&bars[B_TFULL], r & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t st = sb + s * STAGE_BYTES;
                const uint32_t tb = sb + OFF_TB + (r & 1) * 8192;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    umma_bf16(tmem + TM_WT, sdesc(st + 8192 + j * 2048, 16384, 1024),
                              sdesc(tb + j * 32, 16, 1024), i_tt, j > 0);
                if (has_v) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_bf16(tmem + TM_ZU + (r & 1) * 64, sdesc(st + 32768 + j * 2048, 8192, 1024),
                                  sdesc(tb + j * 32, 16, 1024), i_tt, j > 0);
                }
                umma_commit(&bars[B_WUFULL]);
                return true;
            };
            ok = m1(0) && m23(0);
            for (int r = 0; ok && r < nch; ++r) {
                const int s = r & 1;
                const uint32_t st = sb + s * STAGE_BYTES;
                if (!mbar_wait(&bars[B_WFULL], r & 1, abort_flag) ||
                    !mbar_wait(&bars[B_SBF], r & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                // Z^T = U^T - S^T W^T
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t off = (j >> 2) * 16384 + (j & 3) * 32;
                    const uint32_t woff = (j >> 2) * 8192 + (j & 3) * 32;
                    umma_bf16(tmem + TM_ZU + (r & 1) * 64, sdesc(sb + OFF_SBF + off, 16, 1024),
                              sdesc(sb + OFF_WB + woff, 16, 1024), i_c1a, has_v ? 1u : (j > 0 ? 1u : 0u));
                }
                umma_commit(&bars[B_C1A]);
                if (HAS_Q) {
                    if (!mbar_wait(&bars[B_OFREE], r & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    // O^T = S^T Q^T
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t off = (j >> 2) * 16384 + (j & 3) * 32;
                        umma_bf16(tmem + TM_O, sdesc(sb + OFF_SBF + off, 16, 1024),
                                  sdesc(st + (j >> 2) * 16384 + (j & 3) * 32, 16, 1024), i_c1b, j > 0);
                    }
                }
                if (r + 1 < nch) {
                    if (!mbar_wait(&bars[B_GFREE], r & 1, abort_flag) || !m1(r + 1)) { ok = false; break; }
                }
                if (!mbar_wait(&bars[B_ZFULL], r & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                // S^T += Z^T K
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    umma_bf16(tmem + TM_S, sdesc(sb + OFF_ZB + j * 32, 16, 1024),
                              sdesc(st + 8192 + j * 2048, 16384, 1024), i_c3, 1u);
                umma_commit(&bars[B_SFULL]);
                if (HAS_Q) {
                    // O^T += Z^T P^T
                    const uint32_t pb = sb + OFF_PB + (r & 1) * 8192;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_bf16(tmem + TM_O, sdesc(sb + OFF_ZB + j * 32, 16, 1024),
                                  sdesc(pb + j * 32, 16, 1024), i_c2, 1u);
                    umma_commit(&bars[B_OFULL]);
                }
                umma_commit(&bars[B_EMPTY + s]);
                if (r + 1 < nch && !m23(r + 1)) { ok = false; break; }
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ chunk-parallel epilogue
        const int q = warp - 8, wt = threadIdx.x - 256;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const float* bg = p.beta + it.b * p.b_sb + it.head * p.b_sh;
        for (int r = 0; r < nch; ++r) {
            float* bc = betas + (r & 1) * 64;
            const int t0 = it.tok0 + r * kChunk;
            if (wt < 64) bc[wt] = (t0 + wt < it.tok1) ? bg[(int64_t)(t0 + wt) * p.b_st] : 0.f;
            named_sync(1, 128);
            mbar_wait(&bars[B_GFULL], r & 1, abort_flag);
            tc_fence_after();
            {
                uint32_t v[32];
                if (q >= 2) {
                    // key rows: A = B L (strict lower), blocked
                    const int i = 32 * (q - 2) + lane, bi = i >> 4, ii = i & 15;
                    const float bet = bc[i];
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        tmem_ld32(tmem + lane_base + TM_G + 32 * half, v);
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int j = 32 * half + jj, bj = j >> 4;
                            if (bj < bi)
                                Ablk[bidx(bi, bj) * BLK_FLOATS + ii * BLK_LD + (j & 15)] =
                                    bet * __uint_as_float(v[jj]);
                            else if (bj == bi)
                                Ablk[bidx(bi, bj) * BLK_FLOATS + ii * BLK_LD + (j & 15)] =
                                    j < i ? bet * __uint_as_float(v[jj]) : 0.f;
                        }
                    }
                } else if (HAS_Q) {
                    // query rows: P = (Q K^T) o M_c (inclusive), bf16
                    const int i = 32 * q + lane;
                    uint8_t* pb = smem + OFF_PB + (r & 1) * 8192;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        tmem_ld32(tmem + lane_base + TM_G + 32 * half, v);
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj)
                            if (32 * half + jj > i) v[jj] = 0u;
                        st_row32_bf16(pb, i, 32 * half, v);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[B_GFREE]);
            named_sync(1, 128);
            // diagonal 16 x 16 blocks of N = (I + A)^{-1}: one column per thread
            if (wt < 64) {
                const int blk = wt >> 4, c = wt & 15;
                const float* Ab = Ablk + bidx(blk, blk) * BLK_FLOATS;
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = (i == c) ? 1.f : 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j)
#pragma unroll
                    for (int i = j + 1; i < 16; ++i) x[i] = fmaf(-Ab[i * BLK_LD + j], x[j], x[i]);
                float* Nb = Nblk + bidx(blk, blk) * BLK_FLOATS;
#pragma unroll
                for (int i = 0; i < 16; ++i) Nb[i * BLK_LD + c] = x[i];
            }
            named_sync(1, 128);
            // off-diagonal blocks: N_ij = -N_ii sum_{k=j}^{i-1} A_ik N_kj, by distance i - j
#pragma unroll 1
            for (int dd = 1; dd < 4; ++dd) {
                if (q < 4 - dd) {
                    const int i = q + dd, j = q;
                    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                    for (int kb = j; kb < i; ++kb)
                        mm16(acc, Ablk + bidx(i, kb) * BLK_FLOATS, Nblk + bidx(kb, j) * BLK_FLOATS);
                    float* X = Xs + q * BLK_FLOATS;
                    st16(X, acc, 1.f);
                    __syncwarp();
                    float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                    mm16(acc2, Nblk + bidx(i, i) * BLK_FLOATS, X);
                    st16(Nblk + bidx(i, j) * BLK_FLOATS, acc2, -1.f);
                }
                named_sync(1, 128);
            }
            // T = N diag(beta) -> bf16, swizzled rows
            {
                const int i = wt >> 1, hh = wt & 1, bi = i >> 4;
                uint8_t* tb = smem + OFF_TB + (r & 1) * 8192;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float vals[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = 32 * hh + 8 * cc + e, bj = j >> 4;
                        vals[e] = (j <= i) ? Nblk[bidx(bi, bj) * BLK_FLOATS + (i & 15) * BLK_LD + (j & 15)] * bc[j]
                                           : 0.f;
                    }
                    uint4 u;
                    u.x = pack_bf16(vals[0], vals[1]);
                    u.y = pack_bf16(vals[2], vals[3]);
                    u.z = pack_bf16(vals[4], vals[5]);
                    u.w = pack_bf16(vals[6], vals[7]);
                    *reinterpret_cast<uint4*>(tb + swz128(i, 32 * hh + 8 * cc)) = u;
                }
            }
            fence_async_smem();
            mbar_arrive(&bars[B_TFULL]);
            // W^T (TMEM) -> W (bf16, rows = tokens) once the previous W is consumed
            if (r >= 1) mbar_wait(&bars[B_C1A], (r - 1) & 1, abort_flag);
            mbar_wait(&bars[B_WUFULL], r & 1, abort_flag);
            tc_fence_after();
            {
                const int dk = 32 * q + lane;
                const int atom = dk >> 6;
                const int pc = (dk & 63) & ~1;  // even column of the pair
                uint32_t v[32];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    tmem_ld32(tmem + lane_base + TM_WT + 32 * half, v);
#pragma unroll
                    for (int tt = 0; tt < 32; tt += 2) {
                        const float v0 = __uint_as_float(v[tt]), v1 = __uint_as_float(v[tt + 1]);
                        const float send = (lane & 1) ? v0 : v1;
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                        const int row = 32 * half + tt + (lane & 1);
                        const uint32_t pk = (lane & 1) ? pack_bf16(recv, v1) : pack_bf16(v0, recv);
                        *reinterpret_cast<uint32_t*>(Wb + atom * 8192 + swz128(row, pc)) = pk;
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_WFULL]);
        }
    } else {
        // ------------------------------------------------------------ chain epilogue
        const int wq = warp & 3, h = warp >> 2;
        const int d = 32 * wq + lane;  // d_v row of S^T, Z^T, O^T
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        {
            uint32_t v[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int a = 64 * h + 32 * half + c;
                    float x = 0.f;
                    if (x_in) x = x_in[(int64_t)a * D + d];
                    else if (identity) x = (a == d) ? 1.f : 0.f;
                    v[c] = __float_as_uint(x);
                }
                if (nch == 0) {
                    if (x_out)
                        for (int c = 0; c < 32; ++c) x_out[(int64_t)(64 * h + 32 * half + c) * D + d] = __uint_as_float(v[c]);
                } else {
                    tmem_st32(tmem + lane_base + TM_S + 64 * h + 32 * half, v);
                    st_row32_bf16(Sbf + h * 16384, d, 32 * half, v);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&bars[B_SBF]);
        if (HAS_Q) mbar_arrive(&bars[B_OFREE]);
        __nv_bfloat16* og = static_cast<__nv_bfloat16*>(p.o) + it.b * p.o_sb + it.head * p.o_sh;
        for (int r = 0; r < nch; ++r) {
            uint32_t v[32];
            // Z^T -> bf16 operand
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_C1A], r & 1, abort_flag))) break;
            tc_fence_after();
            tmem_ld32(tmem + lane_base + TM_ZU + (r & 1) * 64 + 32 * h, v);
            st_row32_bf16(Zb, d, 32 * h, v);
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_ZFULL]);
            // S^T -> bf16 operand (and fp32 out after the last chunk)
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL], r & 1, abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld32(tmem + lane_base + TM_S + 64 * h + 32 * half, v);
                st_row32_bf16(Sbf + h * 16384, d, 32 * half, v);
                if (r == nch - 1 && x_out) {
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        x_out[(int64_t)(64 * h + 32 * half + c) * D + d] = __uint_as_float(v[c]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_SBF]);
            // O^T -> out (rows = tokens), two d_v columns per 4-byte store
            if (HAS_Q) {
                if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_OFULL], r & 1, abort_flag))) break;
                tc_fence_after();
                tmem_ld32(tmem + lane_base + TM_O + 32 * h, v);
                tc_fence_before();
                mbar_arrive(&bars[B_OFREE]);
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
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicExch(p.err, kErrTimeout);
}

}  // namespace tc
}  // namespace dn
