// Shared definitions of the chunkwise DeltaNet kernels (sm_100a).
//
// Notation follows "Linear Attention, Visualized" (DeltaNet section), row-vector
// convention: a chunk holds C = 64 tokens; K_r, Q_r are C x d_k, V_r is C x d_v;
// the state S is d_k x d_v and is read as k S / q S.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace dn {

constexpr int kChunk = 64;       // C
constexpr int kThreads = 256;    // 8 warps per CTA
constexpr int kWarps = kThreads / 32;
constexpr int kMaxSlots = 4096;  // segment-map slots (P, H, start state) per call
// workspace bytes per (chunk, head) written by the UT pre-pass: T tile, then P tile, and for
// Gated DeltaNet a third tile T' = T diag(lambda[1:l]) (at kUnitT2), the decayed queries
// Q<- = diag(lambda[1:l]) Q as two 64-channel boxes (at kUnitQL) and the chunk's row factors
// F (at kUnitF: lambda[l+1:C] for rows l = 0..63, then lambda[1:C]), padded to 1 KB
constexpr int kUnitBytes = 16384;
constexpr int kUnitT2 = 16384, kUnitQL = 24576, kUnitF = 40960, kUnitFBytes = 512;
constexpr int kUnitBytesGated = 41984;
__host__ __device__ constexpr int unit_bytes(bool gated) { return gated ? kUnitBytesGated : kUnitBytes; }

// Gated DeltaNet: the log decays g of tokens [t, t + 64) of one (batch row, head), two
// per lane: lane l reads tokens t + 2 l and t + 2 l + 1 (tokens at or past `t_end` count
// as g = 0, a = 1).
__device__ __forceinline__ float2 gate_load(const float* gbase, int64_t g_st, int t, int t_end) {
    const int j = 2 * (threadIdx.x & 31);
    return make_float2(t + j < t_end ? gbase[(int64_t)(t + j) * g_st] : 0.f,
                       t + j + 1 < t_end ? gbase[(int64_t)(t + j + 1) * g_st] : 0.f);
}
// Their inclusive prefix sums over the chunk: lane l gets c[2 l] and c[2 l + 1]
// (c_j = g_0 + ... + g_j).  A whole warp.
__device__ __forceinline__ float2 gate_scan(float2 g) {
    const int lane = threadIdx.x & 31;
    float s = g.x + g.y;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
    }
    // s = c[2 lane + 1]; c[2 lane] = s - g1
    return make_float2(s - g.y, s);
}
// Their total c_63 on every lane.  A whole warp.
__device__ __forceinline__ float gate_sum(float2 g) {
    float s = g.x + g.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}
__device__ __forceinline__ float2 gate_prefix(const float* gbase, int64_t g_st, int t, int t_end) {
    return gate_scan(gate_load(gbase, g_st, t, t_end));
}
constexpr int kAutoMaxSlots = 592;  // slots the automatic schedule may use (4 x 148)

// Device error flag values (match dn_status).
constexpr int kErrSeqlens = 6;
constexpr int kErrTimeout = 7;

// A unit of work: one run of whole chunks of one (sequence, head) chain.
//   b       batch row holding the tokens (0 for packed varlen input)
//   seq     sequence index n (state row)
//   head    head index h
//   tok0/1  token range [tok0, tok1) within batch row b
//   g, G    segment index and segment count of the chain
//   slot    first workspace slot of the chain (segments 0..G-2 use slot+g)
//   cbase   global index of the run's first chunk (chunks are numbered per
//           sequence in order, all heads sharing one number)
struct Item {
    int b, seq, head, tok0, tok1, g, G, slot, cbase;
};

enum SegMode : int {
    kModeOut = 0,    // boundary pass with output: start state -> O, end state
    kModeEnd = 1,    // first segment: end state from the true initial state (no output)
    kModeH = 2,      // zero-start local writes H_g of a segment
    kModeP = 3,      // transition product P_g of a segment (state is d_k x d_k, starts at I)
    kModeHP = 4,     // both maps of a segment, H_g and P_g, in one item
};

// How work items are enumerated.
//  dense:  B x H chains of n_chunks chunks each, G segments of s chunks.
//  list:   items written by the device scheduler (packed varlen input).
struct Sched {
    int list;           // 0 = dense, 1 = list
    int B, T, H;        // dense shape
    int n_chunks, G, s; // dense segmentation: G runs of s chunks (run 0: s0, see below)
    int s0;             // dense: chunks of run 0 (0: s); the last run takes the remainder
    int e_in_c;         // dense: run 0's end state comes from the boundary pass (no E items)
    int c_part;         // dense boundary items: 0 all runs, 1 run 0 only, 2 runs 1..G-1
    const Item* itemsC;     // list: boundary-pass items
    const Item* itemsA;     // list: summary items; Item.g carries mode in bits 16+
    const Item* itemsScan;  // list: one per chain with G >= 2
    const int* counts;      // list: [nC, nA, nScan, total chunks]
    const int* cumchunks;   // list: [N + 1] first global chunk index of each sequence
    const int* cu;          // list: cu_seqlens [N + 1]
    int N;                  // list: number of sequences
    int cu_mul;             // list: rows per token of cu_seqlens (Gated Delta Product: n_h)
};

struct Params {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    const float* beta;
    const float* g;      // Gated DeltaNet: log decay ln a_t [B, T, H]; null for DeltaNet
    const float* s0;     // may be null
    float* sT;           // may be null
    int64_t q_sb, q_st, q_sh;
    int64_t k_sb, k_st, k_sh;
    int64_t v_sb, v_st, v_sh;
    int64_t o_sb, o_st, o_sh;
    int64_t b_sb, b_st, b_sh;
    int64_t g_sb, g_st, g_sh;
    // Gated Delta Product: delta-rule writes per token (<= 1: one).  Token ranges of the
    // items then count virtual steps m (k, v, beta rows); q, g and o rows are tokens
    // m / nh, read (q) and written (o) at the last step of a token, g at its first.
    int nh;
    // Chunk-start states for a backward pass: the state entering every chunk, fp32
    // [rows][H][d_k][d_v] at row (global chunk index), or null.
    float* cs;
    int64_t cs_sc, cs_sh, cs_rows;
    int64_t s0_sn, s0_sh;
    int64_t sT_sn, sT_sh;
    float* wsP;          // [slots][d_k][d_k]
    float* wsH;          // [slots][d_k][d_v]
    float* wsS;          // [slots][d_k][d_v] start states of segments 1..G-1
    uint8_t* wsT;        // [chunks * H] UT factors T (bf16 64 x 64, 128-byte swizzled rows)
    int* err;            // device error flag
    // Bounded waits: the time after which a wait gives up (0: 2 s).  stall_chunk > 0 makes
    // the tensor-core boundary kernel's chain issuer wait, at chunk stall_chunk - 1 of each
    // run, on a barrier that nothing completes, so that the time-out path (give up, drain,
    // report DN_ERR_TIMEOUT) can be tested with no fault; 0 in normal calls.
    unsigned long long wait_ns;
    int stall_chunk;
    Sched sched;
};

// ---- schedule decoding --------------------------------------------------------

__device__ __forceinline__ void dense_chain_item(const Sched& s, int chain, int g, Item& it) {
    it.b = chain / s.H;
    it.seq = it.b;
    it.head = chain % s.H;
    it.G = s.G;
    it.g = g;
    // run g covers chunks [c0, c1): run 0 the first s0, every later run s (the last one
    // whatever remains)
    const int s0 = s.s0 > 0 ? s.s0 : s.s;
    const int c0 = g == 0 ? 0 : s0 + (g - 1) * s.s;
    const int c1 = g == 0 ? s0 : s0 + g * s.s;
    it.tok0 = c0 * kChunk;
    const long long e = (long long)c1 * kChunk;
    it.tok1 = e < s.T ? (int)e : s.T;
    if (g == s.G - 1) it.tok1 = s.T;
    it.slot = chain * (s.G - 1);
    it.cbase = it.b * s.n_chunks + c0;
}

__device__ __forceinline__ int count_C(const Sched& s) {
    if (s.list) return s.counts[0];
    const int runs = s.c_part == 0 ? s.G : (s.c_part == 1 ? 1 : s.G - 1);
    return s.B * s.H * runs;
}
__device__ __forceinline__ int count_A(const Sched& s) {
    return s.list ? s.counts[1] : (s.G >= 2 ? s.B * s.H * (s.G - 1 - s.e_in_c) : 0);
}
__device__ __forceinline__ int count_scan(const Sched& s) {
    return s.list ? s.counts[2] : (s.G >= 2 ? s.B * s.H : 0);
}

__device__ __forceinline__ Item item_C(const Sched& s, int i) {
    Item it;
    if (s.list) return s.itemsC[i];
    if (s.c_part == 0) dense_chain_item(s, i / s.G, i % s.G, it);
    else if (s.c_part == 1) dense_chain_item(s, i, 0, it);
    else dense_chain_item(s, i / (s.G - 1), 1 + i % (s.G - 1), it);
    return it;
}

// Summary items: per chain, [End(g=0), HP(1), HP(2), ..., HP(G-2)], or without the End
// item when the boundary pass's run-0 item writes run 0's end state (e_in_c).
__device__ __forceinline__ Item item_A(const Sched& s, int i, int& mode) {
    Item it;
    if (s.list) {
        it = s.itemsA[i];
        mode = it.g >> 16;
        it.g &= 0xffff;
        return it;
    }
    const int per = s.G - 1 - s.e_in_c;
    const int chain = i / per, r = i % per + s.e_in_c;
    mode = r == 0 ? kModeEnd : kModeHP;
    dense_chain_item(s, chain, r, it);
    return it;
}

// Chunk-head units of the UT pre-pass: (global chunk, head).
__device__ __forceinline__ int count_chunks(const Sched& s) {
    return s.list ? s.counts[3] : s.B * s.n_chunks;
}

// Token range and batch row of global chunk `id`.
__device__ __forceinline__ void chunk_range(const Sched& s, int id, int& b, int& t0, int& t1) {
    if (!s.list) {
        b = id / s.n_chunks;
        t0 = (id % s.n_chunks) * kChunk;
        t1 = min(s.T, t0 + kChunk);
        return;
    }
    int lo = 0, hi = s.N;  // largest n with cumchunks[n] <= id
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s.cumchunks[mid] <= id) lo = mid;
        else hi = mid;
    }
    b = 0;
    t0 = s.cu[lo] * s.cu_mul + (id - s.cumchunks[lo]) * kChunk;
    t1 = min(s.cu[lo + 1] * s.cu_mul, t0 + kChunk);
}

__device__ __forceinline__ Item item_scan(const Sched& s, int i) {
    Item it;
    if (s.list) return s.itemsScan[i];
    dense_chain_item(s, i, 0, it);
    return it;
}

}  // namespace dn
