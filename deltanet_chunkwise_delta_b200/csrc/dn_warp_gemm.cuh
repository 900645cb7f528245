// Warp-level tile products on shared-memory tiles.
//
// Every tile in shared memory is row-major with an XOR swizzle on 16-byte
// chunks (chunk index ^= row % 8), so that 8 consecutive rows of one column
// chunk fall in distinct banks.  A warp computes a 16 x (8 NT) fp32 block held
// in the accumulator layout of mma.m16n8: thread (g = lane / 4, t = lane % 4)
// owns rows g and g + 8, columns 2t and 2t + 1 of each 16 x 8 tile.
//
// bf16 operands go through ldmatrix + mma.sync (fp32 accumulation); fp32
// operands go through scalar FMAs with the same register layout, so the
// kernels above share one code path for both storage types.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace dn {

template <typename E>
struct Swz {
    static constexpr int V = 16 / sizeof(E);  // elements per 16-byte chunk
    template <int LD>
    __device__ __forceinline__ static int off(int r, int c) {
        static_assert(LD / V >= 8, "tile rows must hold at least 8 chunks");
        return r * LD + (((c / V) ^ (r & 7)) * V) + (c % V);
    }
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// acc[nt] += A[r0 : r0+16, 0 : K] * B[0 : K, n0 + 8 nt : n0 + 8 nt + 8]
//   A(r, k) = AT ? A_tile[k][r] : A_tile[r][k]      (tile width LDA)
//   B(k, n) = BKN ? B_tile[k][n] : B_tile[n][k]     (tile width LDB)
template <int K, int NT, int LDA, bool AT, int LDB, bool BKN>
__device__ __forceinline__ void warp_gemm(float (&acc)[NT][4], const __nv_bfloat16* A, int r0,
                                          const __nv_bfloat16* B, int n0) {
    static_assert(K % 16 == 0 && NT % 2 == 0, "shape");
    using S = Swz<__nv_bfloat16>;
    const int lane = threadIdx.x & 31;
    const int i8 = lane & 7, sel = lane >> 3;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t a[4];
        if (!AT) {
            const int r = r0 + i8 + (sel & 1) * 8, c = k0 + (sel >> 1) * 8;
            ldsm_x4(a, smem_addr(A + S::off<LDA>(r, c)));
        } else {
            const int kr = k0 + i8 + (sel >> 1) * 8, rc = r0 + (sel & 1) * 8;
            ldsm_x4_t(a, smem_addr(A + S::off<LDA>(kr, rc)));
        }
#pragma unroll
        for (int nt = 0; nt < NT; nt += 2) {
            uint32_t b[4];
            const int nb = n0 + nt * 8;
            if (!BKN) {
                const int nr = nb + i8 + (sel >> 1) * 8, kc = k0 + (sel & 1) * 8;
                ldsm_x4(b, smem_addr(B + S::off<LDB>(nr, kc)));
            } else {
                const int kr = k0 + i8 + (sel & 1) * 8, nc = nb + (sel >> 1) * 8;
                ldsm_x4_t(b, smem_addr(B + S::off<LDB>(kr, nc)));
            }
            mma_bf16(acc[nt], a, b[0], b[1]);
            mma_bf16(acc[nt + 1], a, b[2], b[3]);
        }
    }
}

template <int K, int NT, int LDA, bool AT, int LDB, bool BKN>
__device__ __forceinline__ void warp_gemm(float (&acc)[NT][4], const float* A, int r0,
                                          const float* B, int n0) {
    using S = Swz<float>;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int ra = r0 + g, rb = r0 + g + 8;
#pragma unroll 4
    for (int k = 0; k < K; ++k) {
        const float a0 = AT ? A[S::off<LDA>(k, ra)] : A[S::off<LDA>(ra, k)];
        const float a1 = AT ? A[S::off<LDA>(k, rb)] : A[S::off<LDA>(rb, k)];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int c = n0 + nt * 8 + 2 * t;
            const float b0 = BKN ? B[S::off<LDB>(k, c)] : B[S::off<LDB>(c, k)];
            const float b1 = BKN ? B[S::off<LDB>(k, c + 1)] : B[S::off<LDB>(c + 1, k)];
            acc[nt][0] = fmaf(a0, b0, acc[nt][0]);
            acc[nt][1] = fmaf(a0, b1, acc[nt][1]);
            acc[nt][2] = fmaf(a1, b0, acc[nt][2]);
            acc[nt][3] = fmaf(a1, b1, acc[nt][3]);
        }
    }
}

// Store a 16 x (8 NT) accumulator block (rows r0.., cols n0..) into a swizzled
// tile of width LD, multiplied by `scale`.
template <int NT, int LD>
__device__ __forceinline__ void store_frag(__nv_bfloat16* T, int r0, int n0,
                                           const float (&acc)[NT][4], float scale) {
    using S = Swz<__nv_bfloat16>;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int c = n0 + nt * 8 + 2 * t;
        *reinterpret_cast<__nv_bfloat162*>(T + S::off<LD>(r0 + g, c)) =
            __floats2bfloat162_rn(acc[nt][0] * scale, acc[nt][1] * scale);
        *reinterpret_cast<__nv_bfloat162*>(T + S::off<LD>(r0 + g + 8, c)) =
            __floats2bfloat162_rn(acc[nt][2] * scale, acc[nt][3] * scale);
    }
}

template <int NT, int LD>
__device__ __forceinline__ void store_frag(float* T, int r0, int n0, const float (&acc)[NT][4],
                                           float scale) {
    using S = Swz<float>;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int c = n0 + nt * 8 + 2 * t;
        *reinterpret_cast<float2*>(T + S::off<LD>(r0 + g, c)) =
            make_float2(acc[nt][0] * scale, acc[nt][1] * scale);
        *reinterpret_cast<float2*>(T + S::off<LD>(r0 + g + 8, c)) =
            make_float2(acc[nt][2] * scale, acc[nt][3] * scale);
    }
}

template <int NT>
__device__ __forceinline__ void zero_frag(float (&acc)[NT][4]) {
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
}

}  // namespace dn
