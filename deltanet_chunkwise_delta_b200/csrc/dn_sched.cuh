// Segmentation of (sequence, head) chains into runs of chunks.
//
// A chain of n_c chunks is cut into G runs: run 0 of s0 chunks, then runs of s
// chunks (the last one possibly shorter).  Run 0 starts from the true initial
// state; the others need the maps (P_g, H_g) of every run before them ("Context
// Parallelism for DeltaNet", section 3: the chunk update is affine in the
// incoming state, so runs compose).  Work per call:
//   summary pass   run 0: end state; runs 1..G-2: H_g and P_g (one item each)
//   segment scan   start states of runs 1..G-1
//   boundary pass  every run from its start state: outputs, final state
// The run lengths minimise a simple model of the call's duration, with costs
// per chunk relative to one boundary-pass chunk and one CTA per SM
// (waves(n) = ceil(n / SMs)):
//   dense, equal runs (s0 = s):     c * s * waves(runs) + a * s * waves(summary items)
//                                   + scan * (G - 1)
//   dense, run 0 on the boundary    phase 1, run 0 (c per chunk) next to the summary
//   pass next to the summary        items (a per chunk): max(c * s0, a * s) * waves;
//   pass (tensor-core path):        phase 2, runs 1..G-1: c * s * waves; + scan * (G - 1);
//                                   s0 = (a / c) s, so that both parts of phase 1 end together
//   packed input (unequal):         c * max(min(s, longest chain), chunk-heads / SMs)
//                                   + a * max(s, summary chunk-heads / SMs) + scan * (G_max - 1)
#pragma once

#include "dn_common.cuh"

namespace dn {

struct CostModel {
    float c = 1.0f;      // boundary pass, per chunk
    float a = 1.25f;     // summary pass, per chunk (mma.sync path: two chains, no output)
    float scan = 2.0f;   // one step of the segment scan
};
// Summary-pass chunk of the tensor-core path (two chains, k_tc_summary) relative to its
// boundary-pass chunk (measured: 1.9 against 1.5 us per chunk).
constexpr float kTcSummaryCost = 1.25f;

struct SegChoice {
    int s;
    float cost;
    int s0 = 0;          // chunks of run 0 (0: s)
};

// Cost of equal runs of length s for `chains` chains of equal length n_c (dense input,
// every run's end state from the summary pass).
__host__ __device__ inline float dense_cost(const CostModel& m, int chains, int n_c, int s,
                                            int slots) {
    const int G = n_c > 0 ? (n_c + s - 1) / s : 1;
    const long long runs = (long long)chains * G;
    const long long summ = G >= 2 ? (long long)chains * (G - 1) : 0;
    const float wC = (float)((runs + slots - 1) / slots);
    const float wA = (float)((summ + slots - 1) / slots);
    return m.c * min(s, n_c) * wC + m.a * s * wA + m.scan * (G - 1);
}

// The run lengths for `chains` chains of n_c chunks.  With e_in_c, run 0 of a split
// chain is computed once, by its boundary item, which runs next to the summary items
// (G - 1 items per chain in each of the two phases).
inline SegChoice choose_dense(const CostModel& m, int chains, int n_c, int slots,
                              int max_slots, bool e_in_c = false) {
    if (n_c <= 0) return {1, 0.f};
    const auto waves = [&](long long n) { return (float)((n + slots - 1) / slots); };
    SegChoice best{n_c, m.c * n_c * waves(chains)};  // one run per chain
    if (!e_in_c) {
        for (int G = 2; G <= 256 && G <= n_c; ++G) {
            const int s = (n_c + G - 1) / G;
            const int Gs = (n_c + s - 1) / s;
            if ((long long)chains * (Gs - 1) > max_slots) break;
            const float cst = dense_cost(m, chains, n_c, s, slots);
            if (cst < best.cost) best = {s, cst};
        }
        return best;
    }
    const float rho = fminf(1.f, m.a / m.c);
    for (int G = 2; G <= 256 && G <= n_c; ++G) {
        if ((long long)chains * (G - 1) > max_slots) break;
        int s = (int)ceilf((float)n_c / ((float)(G - 1) + rho));
        int s0 = n_c - (G - 1) * s;
        if (s0 < 1) continue;
        const float w = waves((long long)chains * (G - 1));
        const float phase1 = fmaxf(m.c * s0, G >= 3 ? m.a * s : 0.f);
        const float cst = phase1 * w + m.c * s * w + m.scan * (G - 1);
        if (cst < best.cost) best = {s, cst, s0 < s ? s0 : 0};
    }
    return best;
}

// Device scheduler for packed variable-length input (one CTA of 1024 threads).
// Validates cu_seqlens, picks s (unless forced), orders sequences longest
// first and writes the three item lists and their counts.
// Also numbers the chunks of all sequences in input order (cumchunks[N + 1],
// counts[3] = total) for the UT pre-pass.
// Scratch: nc[N], order[N], offs[N][4].
// cu_mul: token ranges are cu[n] * cu_mul (Gated Delta Product: cu counts tokens, the
// items count virtual steps, cu_mul per token); T counts the same units as the items.
__global__ void __launch_bounds__(1024) k_schedule(const int* __restrict__ cu, int cu_mul, int N,
                                                   int T, int H, int forced_s, int max_slots,
                                                   int slots, CostModel m, Item* itemsC,
                                                   Item* itemsA, Item* itemsScan, int* counts,
                                                   int* nc, int* order, int4* offs, int* cumchunks,
                                                   int* err) {
    __shared__ int s_err, s_lmax;
    __shared__ unsigned long long s_total;
    __shared__ float s_cost[64];
    __shared__ int s_s;
    __shared__ int4 s_warp[32];
    __shared__ int4 s_carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        s_err = 0;
        s_lmax = 0;
        s_total = 0;
        s_carry = make_int4(0, 0, 0, 0);
    }
    __syncthreads();
    if (N > 0 && tid == 0 && (cu[0] != 0 || (long long)cu[N] * cu_mul != T)) s_err = 1;
    for (int n = tid; n < N; n += blockDim.x) {
        const long long a64 = (long long)cu[n] * cu_mul, e64 = (long long)cu[n + 1] * cu_mul;
        if (e64 < a64 || a64 < 0 || e64 > T) atomicOr(&s_err, 1);
        const int L = e64 > a64 && e64 <= T && a64 >= 0 ? (int)(e64 - a64) : 0;
        const int c = (L + kChunk - 1) / kChunk;
        nc[n] = c;
        atomicMax(&s_lmax, c);
        atomicAdd(&s_total, (unsigned long long)c);
    }
    __syncthreads();
    if (s_err) {
        if (tid == 0) {
            counts[0] = counts[1] = counts[2] = counts[3] = 0;
            atomicExch(err, kErrSeqlens);
        }
        return;
    }
    const int lmax = s_lmax;

    // ---- cumchunks: exclusive prefix of nc in input order
    for (int base = 0; base < N; base += blockDim.x) {
        const int pos = base + tid;
        const int v = pos < N ? nc[pos] : 0;
        int inc = v;
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += x;
        }
        if (lane == 31) s_warp[warp].x = inc;
        __syncthreads();
        if (warp == 0) {
            int t = s_warp[lane].x;
            for (int o = 1; o < 32; o <<= 1) {
                const int x = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += x;
            }
            s_warp[lane].x = t;
        }
        __syncthreads();
        const int before = s_carry.x + (warp > 0 ? s_warp[warp - 1].x : 0);
        if (pos < N) cumchunks[pos] = before + inc - v;
        __syncthreads();
        if (tid == blockDim.x - 1) s_carry.x += s_warp[31].x;
        __syncthreads();
    }
    if (tid == 0) {
        cumchunks[N] = s_carry.x;
        counts[3] = s_carry.x;
        s_carry.x = 0;
    }
    __syncthreads();

    // ---- run length
    if (forced_s > 0) {
        if (tid == 0) s_s = forced_s;
    } else {
        for (int k = warp; k < 64; k += 32) {
            const int s = lmax > 0 ? (lmax + k) / (k + 1) : 1;
            long long extra = 0, wA = 0;
            int gmax = 1;
            for (int n = lane; n < N; n += 32) {
                const int c = nc[n];
                const int G = c > 0 ? (c + s - 1) / s : 1;
                extra += G - 1;
                if (G >= 2) wA += G - 1;
                gmax = max(gmax, G);
            }
            for (int o = 16; o > 0; o >>= 1) {
                extra += __shfl_xor_sync(0xffffffffu, extra, o);
                wA += __shfl_xor_sync(0xffffffffu, wA, o);
                gmax = max(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
            }
            if (lane == 0) {
                float cst = 3.0e38f;
                if ((long long)H * extra <= max_slots) {
                    const double work = (double)H * (double)s_total;
                    cst = m.c * fmaxf((float)min(s, max(lmax, 1)), (float)(work / slots));
                    if (wA > 0)
                        cst += m.a * fmaxf((float)s, (float)((double)H * wA * s / slots));
                    cst += m.scan * (gmax - 1);
                }
                s_cost[k] = cst;
            }
        }
        __syncthreads();
        if (tid == 0) {
            int best = 0;
            for (int k = 1; k < 64; ++k)
                if (s_cost[k] < s_cost[best]) best = k;
            s_s = lmax > 0 ? (lmax + best) / (best + 1) : 1;
        }
    }
    __syncthreads();
    const int s = s_s;

    // ---- order sequences longest first (stable); identity order for very large N
    for (int n = tid; n < N; n += blockDim.x) {
        if (N <= 4096) {
            const int c = nc[n];
            int rank = 0;
            for (int j = 0; j < N; ++j) {
                const int cj = nc[j];
                rank += (cj > c) || (cj == c && j < n);
            }
            order[rank] = n;
        } else {
            order[n] = n;
        }
    }
    __syncthreads();

    // ---- exclusive prefix sums over ordered sequences: (C items, A items, scan items, slots)
    for (int base = 0; base < N; base += blockDim.x) {
        const int pos = base + tid;
        int4 v = make_int4(0, 0, 0, 0);
        if (pos < N) {
            const int c = nc[order[pos]];
            const int G = c > 0 ? (c + s - 1) / s : 1;
            v = make_int4(H * G, G >= 2 ? H * (G - 1) : 0, G >= 2 ? H : 0, H * (G - 1));
        }
        int4 inc = v;
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, inc.x, o);
            const int y = __shfl_up_sync(0xffffffffu, inc.y, o);
            const int z = __shfl_up_sync(0xffffffffu, inc.z, o);
            const int w = __shfl_up_sync(0xffffffffu, inc.w, o);
            if (lane >= o) { inc.x += x; inc.y += y; inc.z += z; inc.w += w; }
        }
        if (lane == 31) s_warp[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            int4 t = s_warp[lane];
            for (int o = 1; o < 32; o <<= 1) {
                const int x = __shfl_up_sync(0xffffffffu, t.x, o);
                const int y = __shfl_up_sync(0xffffffffu, t.y, o);
                const int z = __shfl_up_sync(0xffffffffu, t.z, o);
                const int w = __shfl_up_sync(0xffffffffu, t.w, o);
                if (lane >= o) { t.x += x; t.y += y; t.z += z; t.w += w; }
            }
            s_warp[lane] = t;  // inclusive over warps
        }
        __syncthreads();
        int4 before = s_carry;
        if (warp > 0) {
            const int4 pw = s_warp[warp - 1];
            before.x += pw.x; before.y += pw.y; before.z += pw.z; before.w += pw.w;
        }
        if (pos < N)
            offs[pos] = make_int4(before.x + inc.x - v.x, before.y + inc.y - v.y,
                                  before.z + inc.z - v.z, before.w + inc.w - v.w);
        __syncthreads();
        if (tid == blockDim.x - 1) {
            const int4 tot = s_warp[31];
            s_carry = make_int4(s_carry.x + tot.x, s_carry.y + tot.y, s_carry.z + tot.z,
                                s_carry.w + tot.w);
        }
        __syncthreads();
    }

    // ---- emit items
    for (int pos = tid; pos < N; pos += blockDim.x) {
        const int n = order[pos];
        const int c = nc[n];
        const int G = c > 0 ? (c + s - 1) / s : 1;
        const int4 o = offs[pos];
        const int a = cu[n] * cu_mul, e = cu[n + 1] * cu_mul;  // validated above
        for (int h = 0; h < H; ++h) {
            const int slot = o.w + h * (G - 1);
            for (int g = 0; g < G; ++g) {
                Item it;
                it.b = 0;
                it.seq = n;
                it.head = h;
                it.tok0 = a + g * s * kChunk;
                it.tok1 = (g == G - 1) ? e : min(e, a + (g + 1) * s * kChunk);
                it.g = g;
                it.G = G;
                it.slot = slot;
                it.cbase = cumchunks[n] + g * s;
                itemsC[o.x + h * G + g] = it;
                if (G >= 2 && g + 1 < G) {
                    Item x = it;
                    x.g = g | ((g == 0 ? kModeEnd : kModeHP) << 16);
                    itemsA[o.y + h * (G - 1) + g] = x;
                }
                if (G >= 2 && g == 0) itemsScan[o.z + h] = it;
            }
        }
    }
    if (tid == 0) {
        // totals = carry after the last tile
        counts[0] = s_carry.x;
        counts[1] = s_carry.y;
        counts[2] = s_carry.z;
    }
}

}  // namespace dn
