// fused_rope_attn.cuh -- rotary position embedding fused into a
// FlashAttention-style forward pass on sm_100a.
//
// What it computes (pages "RoPE fused into attention on Ascend" sec. 3/5,
// "FlashAttention in ops-transformer" tiling + online softmax,
// "DynamicNTKOperation" sin/cos definition, "RoPE, RMSNorm, GQA/MQA" sec. 12):
//   Q' = rope(Q), K' = rope(K)  rotate-half, angles from the cos/sin table
//   out = softmax(Q' K'^T * scale) V, causal (key > query masked) or not,
//   query head h reading kv head h / G.
// The rotated tiles exist only in shared memory; nothing rotated is written
// back to global memory.
//
// A persistent grid (one CTA per SM) takes work items from a counter in the
// workspace.  A work item is two 128-row query tiles that read the same key /
// value tiles -- two query heads of one kv group at the same rows when the
// group size G is even, else two consecutive query tiles of one head (the
// second may be absent at the end of a sequence).  Every key tile is loaded
// and rotated once for both query tiles.  24 warps, 80 registers per thread:
//   warps 0-7  softmax of query tile 0, warps 8-15 of query tile 1.  Warp w
//              covers TMEM lanes (rows) 32 (w % 4) .. + 31 and one 64-key half
//              hf = (w / 4) % 2 of every score tile.  Per key tile, one read
//              of the half in two 32-column chunks: each chunk's maximum is
//              checked against the half's reference maximum (an integer that
//              lags the true maximum by at most 2^8) and its exponentials are
//              taken in the same pass; the two halves then agree on the larger
//              reference at a named barrier, and a raised reference rescales
//              P, l and O by exact powers of two.  P (bf16/fp16) is written
//              over the half's own S columns.  At each item start the group
//              rotates its own query tile; at its end, row sums combined and
//              O / l written out (whole tiles by TMA stores when possible).
//   warps 16-19 RoPE warpgroup: rotates every key tile once (decode: the
//              query tile), in place in the 128B-swizzled shared-memory
//              layout.  Element i and its rotate-half partner i + D/2 sit at
//              the same offset of two swizzle atoms (D = 128) or in chunks c
//              and c ^ 4 of one atom (D = 64).  Angles come from a complex
//              recurrence in registers when the sequence's positions are
//              consecutive, else from cos/sin rows that TMA staged beside the
//              tile.
//   warp 20    TMA producer of the query tiles and the key ring (+ cos/sin
//              rows when needed), and the item fetcher.
//   warp 21    tcgen05 issuer (an elected lane of the converged warp) and TMEM
//              owner.  Order per key tile j: PV_0(j), QK_0(j+1), PV_1(j),
//              QK_1(j+1), where S_i = Q_i' K_j'^T goes to TMEM buffer i and
//              O_i += P_i V_j reads P_i from that same buffer.  MMAs issued by
//              one thread execute in issue order, so QK_i(j+1) overwrites P_i
//              only after PV_i(j) has read it, and S_i(j+1) being complete
//              implies O_i holds PV_i(j).
//   warp 22    TMA producer for the V ring.
//   warp 23    idle (takes part in the block-wide barriers only).
// Completion of every async step is tracked by mbarriers; each wait is bounded.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "rope_sincos.cuh"
#include "sm100_ptx.cuh"

namespace rfa {

constexpr int kBlockM = 128;  // query rows per tile (= TMEM lanes)
constexpr int kBlockN = 128;  // keys per tile
constexpr int kAttnThreads = 768;  // 24 warps: 80 registers per thread
constexpr int kSoftmaxWarps = 16;  // 8 per query tile: 4 TMEM lane groups x 2 column halves
constexpr int kRopeWarp0 = 16;
constexpr int kRopeWarps = 4;      // one RoPE warpgroup
constexpr int kRopeThreads = kRopeWarps * 32;
constexpr int kTmaWarp = 20;       // Q, K (+ cos/sin rows)
constexpr int kMmaWarp = 21;
constexpr int kTmaVWarp = 22;      // V: its own producer, so K prefetch never waits on a V slot
// warp 23 only takes part in the block-wide barriers
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only if the max grows by > 2^8

struct AttnArgs {
    void* out;
    const RopeSeed* seeds;  // [sequences] in the caller's order
    const uint32_t* table;  // [tokens][D/2] cos/sin words (query rows of sequences whose positions are not consecutive)
    int32_t* sched;         // two work counters (next item, CTAs done), zero at launch; the last CTA re-zeroes them
    int32_t layout;  // 0 BNSD, 1 TND
    int32_t B, Hq, Hkv, G;
    int32_t S;       // BNSD sequence length
    int32_t causal;
    int32_t pair_heads;  // 1: an item's query tiles are heads 2p, 2p+1 at one tile (G even); 0: tiles 2p, 2p+1 of one head
    float scale_log2;  // softmax scale * log2(e)
    int32_t n_items;
    // TND: sequences sorted by length, descending; seg_item0[k] = first work item of sequence k
    int32_t nseg;
    int32_t seg_start[16];
    int32_t seg_len[16];
    int32_t seg_tiles[16];
    int32_t seg_item0[17];
    int32_t seg_orig[16];  // caller's index of sorted sequence k
    // decode over a KV cache (kernel instantiated with kDecode): work item =
    // (batch, kv head, split of the cache); the query tile holds the G heads x
    // Sq new tokens of that kv group, rows of q viewed as [B*Hq*Sq, D]
    int32_t dec_Sq;          // new tokens per sequence
    int32_t dec_Smax;        // cache rows per sequence (cache viewed as [B*Smax, Hkv, D])
    int32_t dec_splits;      // splits of each sequence's keys
    int32_t dec_chunk;       // keys per split, a multiple of kBlockN
    int32_t dec_max_len;     // upper bound of kv_lens (host planning)
    const int32_t* kv_lens;  // [B] keys in each sequence's cache, Sq <= len <= dec_max_len
    float* part_o;           // splits > 1: [splits][B*Hq*Sq][D] unnormalised O
    float* part_ml;          // splits > 1: [splits][B*Hq*Sq][2] (running max, row sum)
    // extents, for the checks of the bounds-checked build (RFA_CHECKED)
    int64_t out_elems;       // elements of out
    int32_t ntok;            // tokens of q/k/v and rows of the table (decode: cache rows B * Smax)
    int32_t tma_out;         // 1: the output tensor map (q's geometry) describes out
    // decode: the RoPE warps form the query rows' cos/sin themselves (no table kernel first)
    const int32_t* dec_qpos;           // [B, Sq] positions of the new tokens
    const float* dec_inv;              // [B, D/2] frequencies, or nullptr: dec_inv_host for every sequence
    float dec_inv_host[kMaxHalfHost];  // base^(-2j/D), formed on the host in fp64 and rounded once
};

// Work items of one sequence with nt query tiles.
__host__ __device__ inline int32_t items_per_sequence(int32_t Hq, int32_t nt, bool pair_heads) {
    return pair_heads ? (Hq / 2) * nt : Hq * ((nt + 1) / 2);
}

template <int D>
struct AttnCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kAtoms = D / 64;                 // 128-byte swizzle atoms across a row
    static constexpr int kAtomBytes = kBlockM * 128;      // one atom column of a 128-row tile
    static constexpr int kTileBytes = kBlockM * D * 2;    // Q, K or V tile
    static constexpr int kTabBytes = kBlockM * D * 2;     // cos/sin rows of a tile: D/2 fp16 cos + D/2 fp16 sin
    static constexpr int kTabBoxes = D / 64;              // 128-byte boxes of 32 (cos, sin) pairs
    static constexpr int kStages = (D == 64) ? 4 : 2;     // K ring and V ring
    static constexpr int kTStages = (D == 64) ? 4 : 1;    // cos/sin rows of key tiles (positions not consecutive)
    static constexpr int kOffQ = 0;                       // two query tiles
    static constexpr int kOffK = kOffQ + 2 * kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kOffT = kOffV + kStages * kTileBytes;
    static constexpr int kOffBar = kOffT + kTStages * kTabBytes;
    // barrier indices
    static constexpr int kBarQFull = 0;  // the item's query tiles landed (decode: and their cos/sin rows)
    static constexpr int kBarQReady = 1; // 2: query tile i rotated (its 8 softmax warps; decode: the RoPE warps, tile 0)
    static constexpr int kBarQEmpty = 3; // the item's last QK MMAs are done: the query slots may be reloaded
    static constexpr int kBarItemFull = 4;   // 2: item index published in the slot
    static constexpr int kBarItemEmpty = 6;  // 2: every consumer warp has read the slot
    static constexpr int kBarKFull = 8;
    static constexpr int kBarVFull = kBarKFull + kStages;
    static constexpr int kBarKReady = kBarVFull + kStages;
    static constexpr int kBarKEmpty = kBarKReady + kStages;
    static constexpr int kBarVEmpty = kBarKEmpty + kStages;
    static constexpr int kBarSFull = kBarVEmpty + kStages;  // 2: S_i complete (and every earlier MMA)
    static constexpr int kBarPFull = kBarSFull + 2;         // 2: P_i written, O_i rescaled (8 warp arrivals)
    static constexpr int kBarOFull = kBarPFull + 2;         // 2: last PV_i complete
    static constexpr int kBarMmaFin = kBarOFull + 2;
    static constexpr int kNumBars = kBarMmaFin + 1;
    static constexpr int kOffAbort = kOffBar + 8 * kNumBars;
    static constexpr int kOffTmemSlot = kOffAbort + 16;
    static constexpr int kOffItem = kOffTmemSlot + 16;  // ItemSlot [2]: the item ring
    static constexpr int kOffXchg = kOffItem + 128;     // float [2 query tiles][2 column halves][128 rows]
    // The dynamic shared-memory window starts 1024-byte aligned on sm_100 (the
    // kernel checks it), so no alignment slack is requested.
    static constexpr int kSmemBytes = kOffXchg + 2 * 2 * kBlockM * 4;
    // TMEM columns: S_0, S_1 (P_i over the first 64 columns of S_i), O_0, O_1
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0;      // S_i at 128 i
    static constexpr uint32_t kColO = 256;    // O_i at 256 + D i
    static_assert(kColO + 2 * D <= kTmemCols, "TMEM budget");
    static_assert(kStages >= 2 && kTabBytes == kTileBytes, "decode stages its query rows' cos/sin in a query slot");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct WorkItem {
    int32_t qrow0;  // decode: first row of the query tile in q viewed as [B*Hq*Sq, D]
    int32_t split;  // decode: split index
    int32_t orig;   // sequence index in the caller's order
    int32_t tok0;   // first token of the sequence (BNSD: seq * S)
    int32_t seq;    // BNSD batch index / TND sorted sequence index
    int32_t L;      // sequence length
    int32_t kvh;    // kv head read by both query tiles
    int32_t h[2];   // query heads
    int32_t qt[2];  // query tile indices within the sequence; qt[1] < 0: no second tile
};

// Decode: item x = (sequence, kv head, split), splits of one kv group adjacent.
__device__ __forceinline__ WorkItem decode_item_kv(const AttnArgs& a, int32_t x) {
    WorkItem w;
    w.split = x % a.dec_splits;
    const int32_t bk = x / a.dec_splits;
    w.kvh = bk % a.Hkv;
    w.seq = bk / a.Hkv;
    w.orig = w.seq;
    w.h[0] = w.h[1] = w.kvh * a.G;
    w.qt[0] = 0;
    w.qt[1] = -1;
    w.qrow0 = (w.seq * a.Hq + w.kvh * a.G) * a.dec_Sq;
    const int32_t k0 = w.split * a.dec_chunk;
    const int32_t len = min(max(a.kv_lens[w.seq], 0), a.dec_Smax);
    w.tok0 = w.seq * a.dec_Smax + k0;  // first key of the split in the cache
    w.L = max(0, min(len - k0, a.dec_chunk));
    return w;
}

// BNSD: heads (head pairs when G is even) are taken in groups of
// kOrderGroup; within a group, items run longest first across its heads (a
// list schedule near its lower bound on causal masks, where items range from
// 1 to S/128 key tiles), and a group's K/V stays in L2 while its items run.
// Packed sequences: longest sequence first, the same grouped longest-first
// order over the heads within a sequence.
constexpr int kOrderGroup = 16;
__device__ __forceinline__ WorkItem decode_item(const AttnArgs& a, int32_t x) {
    WorkItem w;
    w.qrow0 = 0;
    w.split = 0;
    int32_t nt, r;
    const bool ph = a.pair_heads != 0;
    if (a.layout == 0) {
        nt = (a.S + kBlockM - 1) / kBlockM;
        const int32_t per_unit = ph ? nt : (nt + 1) / 2;  // items of one head (pair)
        const int32_t units_seq = ph ? a.Hq / 2 : a.Hq;   // head (pair) units per sequence
        const int32_t units = a.B * units_seq;
        const int32_t g = x / (kOrderGroup * per_unit);
        const int32_t rg = x - g * kOrderGroup * per_unit;
        const int32_t ng = min(kOrderGroup, units - g * kOrderGroup);  // units in this group
        const int32_t rank = rg / ng;                                 // 0: each unit's longest item
        const int32_t u = g * kOrderGroup + (rg - rank * ng);
        w.seq = u / units_seq;
        w.orig = w.seq;
        w.tok0 = w.seq * a.S;
        w.L = a.S;
        // unit u's rank-th item in the per-sequence numbering below (longest first)
        r = (u - w.seq * units_seq) * per_unit + rank;
    } else {
        int32_t s = 0;
        while (s + 1 < a.nseg && x >= a.seg_item0[s + 1]) ++s;
        const int32_t rs = x - a.seg_item0[s];
        nt = a.seg_tiles[s];
        w.seq = s;
        w.orig = a.seg_orig[s];
        w.tok0 = a.seg_start[s];
        w.L = a.seg_len[s];
        // within the sequence, the same grouped longest-first order over its heads
        const int32_t per_unit = ph ? nt : (nt + 1) / 2;
        const int32_t units = ph ? a.Hq / 2 : a.Hq;
        const int32_t g = rs / (kOrderGroup * per_unit);
        const int32_t rg = rs - g * kOrderGroup * per_unit;
        const int32_t ng = min(kOrderGroup, units - g * kOrderGroup);
        const int32_t rank = rg / ng;
        r = (g * kOrderGroup + (rg - rank * ng)) * per_unit + rank;
    }
    if (ph) {
        const int32_t hp = r / nt;
        const int32_t qt = nt - 1 - (r - hp * nt);
        w.h[0] = 2 * hp;
        w.h[1] = 2 * hp + 1;
        w.qt[0] = qt;
        w.qt[1] = qt;
    } else {
        const int32_t np = (nt + 1) / 2;
        const int32_t h = r / np;
        const int32_t p = np - 1 - (r - h * np);
        w.h[0] = h;
        w.h[1] = h;
        w.qt[0] = 2 * p;
        w.qt[1] = (2 * p + 1 < nt) ? 2 * p + 1 : -1;
    }
    w.kvh = w.h[0] / a.G;
    return w;
}

// Checked build: a work item's indices lie inside the problem.
__device__ __forceinline__ bool item_in_bounds(const AttnArgs& a, const WorkItem& w, bool decode) {
    if (decode)
        return in_bounds(w.seq >= 0 && w.seq < a.B && w.kvh >= 0 && w.kvh < a.Hkv && w.split >= 0 &&
                         w.split < a.dec_splits && w.qrow0 >= 0 &&
                         static_cast<int64_t>(w.qrow0) + a.G * a.dec_Sq <= static_cast<int64_t>(a.B) * a.Hq * a.dec_Sq &&
                         w.tok0 >= 0 && static_cast<int64_t>(w.tok0) + w.L <= a.ntok);
    const int32_t nseq = a.layout == 0 ? a.B : a.nseg;
    return in_bounds(w.seq >= 0 && w.seq < nseq && w.orig >= 0 && w.orig < a.B && w.h[0] >= 0 && w.h[1] < a.Hq &&
                     w.kvh >= 0 && w.kvh < a.Hkv && w.h[0] / a.G == w.kvh && w.h[1] / a.G == w.kvh &&
                     w.qt[0] >= 0 && w.qt[0] * kBlockM < w.L && w.qt[1] * kBlockM < w.L && w.L >= 1 &&
                     w.tok0 >= 0 && static_cast<int64_t>(w.tok0) + w.L <= a.ntok);
}

template <bool kFP16>
struct IoT;
template <>
struct IoT<false> {
    static __device__ __forceinline__ float2 unpack(uint32_t u) {
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
    }
    static __device__ __forceinline__ uint64_t unpack2(uint32_t u) {  // exact: bf16 -> fp32 is a shift
        return f2pack(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static constexpr uint32_t kFmt = 1;
};
template <>
struct IoT<true> {
    static __device__ __forceinline__ float2 unpack(uint32_t u) {
        return __half22float2(*reinterpret_cast<const __half2*>(&u));
    }
    static __device__ __forceinline__ uint64_t unpack2(uint32_t u) {
        const float2 f = unpack(u);
        return f2pack(f.x, f.y);
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static constexpr uint32_t kFmt = 0;
};

template <bool kFP16>
__device__ __forceinline__ uint32_t pack2(uint64_t v) {
    const float2 f = f2unpack(v);
    return IoT<kFP16>::pack(f.x, f.y);
}

__device__ __forceinline__ uint64_t h2f2x2(uint32_t u) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u));
    return f2pack(f.x, f.y);
}

// Rotate 8 rotate-half pairs held in two 16-byte chunks (x1: dims i..i+7,
// x2: dims i+D/2..i+D/2+7), two dimensions per packed fp32x2 operation.
// t0/t1 hold, per two dimensions, a word of fp16 cosines then a word of fp16
// sines:  x1' = x1 cos - x2 sin,  x2' = x2 cos + x1 sin.
template <bool kFP16>
__device__ __forceinline__ void rotate8(uint4& x1, uint4& x2, const uint4& t0, const uint4& t1) {
    uint32_t* a = reinterpret_cast<uint32_t*>(&x1);
    uint32_t* b = reinterpret_cast<uint32_t*>(&x2);
    const uint32_t cs[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint64_t X1 = IoT<kFP16>::unpack2(a[k]);
        const uint64_t X2 = IoT<kFP16>::unpack2(b[k]);
        const uint64_t C = h2f2x2(cs[2 * k]);
        const uint64_t S = h2f2x2(cs[2 * k + 1]);
        const uint64_t NS = h2f2x2(cs[2 * k + 1] ^ 0x80008000u);  // -sin, exact
        a[k] = pack2<kFP16>(ffma2(X1, C, fmul2(X2, NS)));
        b[k] = pack2<kFP16>(ffma2(X2, C, fmul2(X1, S)));
    }
}

// Two adjacent pairs at once: word wa holds pair f (x0, x1), wb pair f + 1;
// C and S are packed (cos, sin) of frequencies f and f + 1.  The even and odd
// elements of the two words form packed operands, so one packed operation
// serves both pairs:  x0' = x0 c - x1 s,  x1' = x1 c + x0 s.
template <bool kFP16>
__device__ __forceinline__ void rot_adj2(uint32_t& wa, uint32_t& wb, uint64_t C, uint64_t S) {
    uint64_t X0, X1;
    if constexpr (kFP16) {
        const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&wa));
        const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&wb));
        X0 = f2pack(fa.x, fb.x);
        X1 = f2pack(fa.y, fb.y);
    } else {  // bf16 -> fp32 is a shift
        X0 = f2pack(__uint_as_float(wa << 16), __uint_as_float(wb << 16));
        X1 = f2pack(__uint_as_float(wa & 0xffff0000u), __uint_as_float(wb & 0xffff0000u));
    }
    const float2 r0 = f2unpack(fsub2(fmul2(X0, C), fmul2(X1, S)));  // x0 c - x1 s
    const float2 r1 = f2unpack(ffma2(X1, C, fmul2(X0, S)));         // x1 c + x0 s
    wa = IoT<kFP16>::pack(r0.x, r1.x);
    wb = IoT<kFP16>::pack(r0.y, r1.y);
}

// Rotate 8 adjacent pairs held in two 16-byte chunks (x1: pairs i..i+3, x2:
// pairs i+4..i+7), angles from the same table words as rotate8 (t0: pairs
// i..i+3, t1: pairs i+4..i+7): words (2m, 2m + 1) of a chunk take the table's
// cos word 2m and sin word 2m + 1.
template <bool kFP16>
__device__ __forceinline__ void rotate8_adj(uint4& x1, uint4& x2, const uint4& t0, const uint4& t1) {
    rot_adj2<kFP16>(x1.x, x1.y, h2f2x2(t0.x), h2f2x2(t0.y));
    rot_adj2<kFP16>(x1.z, x1.w, h2f2x2(t0.z), h2f2x2(t0.w));
    rot_adj2<kFP16>(x2.x, x2.y, h2f2x2(t1.x), h2f2x2(t1.y));
    rot_adj2<kFP16>(x2.z, x2.w, h2f2x2(t1.z), h2f2x2(t1.w));
}

// Shared-memory address of logical 16-byte chunk L of row r of a 128-row
// tile: 128B swizzle within 128-row atoms of 8 chunks.
template <int D>
__device__ __forceinline__ uint32_t chunk_addr(uint32_t tile, int32_t r, int32_t L) {
    return tile + static_cast<uint32_t>(L >> 3) * AttnCfg<D>::kAtomBytes + static_cast<uint32_t>(r) * 128u +
           ((static_cast<uint32_t>(L & 7) ^ static_cast<uint32_t>(r & 7)) << 4);
}
// Adjacent pairs at D = 128: a task's chunks 2cp and 2cp + 1 lie in atom 0 for cp < 4 and in
// atom 1 for cp >= 4, at the same bank offsets, so a quarter-warp (the 8 tasks of one row)
// taking the even chunks first would touch every second bank twice.  Tasks with cp >= 4 take
// their two chunks, and with them their two groups of 4 frequencies, in the other order: a
// quarter-warp's first access then covers chunks {0,2,4,6} of atom 0 and {1,3,5,7} of atom 1,
// each bank once.
template <int D, bool kAdj>
__device__ __forceinline__ constexpr bool task_swapped(int cp) {
    return kAdj && D == 128 && cp >= 4;
}
// The two chunks a RoPE task rotates together hold the 8 pairs of frequencies
// 8cp..8cp+7: chunks cp and cp + D/16 (rotate-half) or 2cp and 2cp + 1 (adjacent pairs;
// 2cp + 1 first for a swapped task, whose frequency groups are then 8cp+4.., 8cp..).
template <int D, bool kAdj>
__device__ __forceinline__ void task_chunks(uint32_t tile, int32_t r, int cp, uint32_t& o1, uint32_t& o2) {
    const int sw = task_swapped<D, kAdj>(cp) ? 1 : 0;
    o1 = chunk_addr<D>(tile, r, kAdj ? 2 * cp + sw : cp);
    o2 = chunk_addr<D>(tile, r, kAdj ? 2 * cp + 1 - sw : cp + D / 16);
}
// First frequency of a task's k-th group of 4 (k = 0, 1), in the order its chunks are taken.
template <int D, bool kAdj>
__device__ __forceinline__ int task_freq(int cp, int k) {
    return 8 * cp + 4 * (k ^ (task_swapped<D, kAdj>(cp) ? 1 : 0));
}
// Checked build: a task's row and chunk pair lie inside its 128-row tile.
template <int D>
__device__ __forceinline__ bool task_in_tile(int32_t r, int cp) {
    return in_bounds(r >= 0 && r < kBlockM && cp >= 0 && cp < D / 16);
}

// Rotate the first `rows` rows of a 128-row tile in shared memory with the
// cos/sin rows staged at `tab`.  128B swizzle: 16-byte chunk c of row r sits at
// r*128 + ((c ^ (r&7)) << 4) within its 128-row atom.  The table's atoms hold
// 32 (cos, sin) pairs per row, 4 pairs per chunk.
template <int D, bool kFP16, bool kAdj>
__device__ __forceinline__ void rope_tile(uint32_t tile, uint32_t tab, int32_t rows, int32_t rt) {
    constexpr int kPairsPerRow = D / 16;  // 16-byte chunk pairs per row
    constexpr int kIters = kBlockM * kPairsPerRow / kRopeThreads;
#pragma unroll 1
    for (int it = 0; it < kIters; ++it) {
        const int task = rt + kRopeThreads * it;
        const int r = task / kPairsPerRow;
        const int cp = task % kPairsPerRow;
        if (r >= rows || !task_in_tile<D>(r, cp)) continue;
        const uint32_t sw = static_cast<uint32_t>(r & 7);
        uint32_t o1, o2;
        task_chunks<D, kAdj>(tile, r, cp, o1, o2);
        uint4 t0, t1;
        if constexpr (D == 128) {
            // row layout of the table: chunk cp of atom 0 = pairs 8cp..8cp+3,
            // chunk cp of atom 1 = pairs 8cp+4..8cp+7 (conflict-free for the 8
            // lanes of a quarter-warp, which share a row)
            const uint32_t tb = tab + r * 128 + ((cp ^ sw) << 4);
            const uint32_t ta = task_swapped<D, kAdj>(cp) ? AttnCfg<D>::kAtomBytes : 0u;
            t0 = lds128(tb + ta);
            t1 = lds128(tb + (AttnCfg<D>::kAtomBytes - ta));
        } else {
            const uint32_t tb = tab + r * 128;
            const uint32_t tc = static_cast<uint32_t>(cp * 2);
            t0 = lds128(tb + ((tc ^ sw) << 4));
            t1 = lds128(tb + (((tc + 1) ^ sw) << 4));
        }
        uint4 x1 = lds128(o1), x2 = lds128(o2);
        if constexpr (kAdj)
            rotate8_adj<kFP16>(x1, x2, t0, t1);
        else
            rotate8<kFP16>(x1, x2, t0, t1);
        sts128(o1, x1);
        sts128(o2, x2);
    }
}

// Decode: the cos/sin rows of the query tile's G * Sq rows, formed in the kernel and written
// into the second query slot in the layout that a 128-byte-swizzled copy of the table's rows
// would leave there (rope_tile reads them so): row r of the tile is query row qrow0 + r of q
// viewed as [B*Hq*Sq, D], i.e. new token s of sequence b, at position dec_qpos[b][s].  The
// angles go through the table kernels' reduction and SFU evaluation and are packed the same
// way (fp16 (cos, cos), (sin, sin) word pairs, chunk order permuted for D = 128).  Each thread
// takes the tasks (row, chunk pair) that its own rope_tile call reads afterwards, so the
// rows need no barrier between the writes and the reads.
template <int D>
__device__ __forceinline__ void decode_query_table(uint32_t tab, const AttnArgs& a, int32_t qrow0, int32_t rt) {
    constexpr int kPairsPerRow = D / 16;  // 8-frequency tasks per row
    constexpr int kIters = kBlockM * kPairsPerRow / kRopeThreads;
    constexpr int kHalf = D / 2;
    const int32_t rows = a.G * a.dec_Sq;
    const int32_t per_seq = a.Hq * a.dec_Sq;  // query rows of one sequence
#pragma unroll 1
    for (int it = 0; it < kIters; ++it) {
        const int task = rt + kRopeThreads * it;
        const int32_t r = task / kPairsPerRow;
        const int c = task % kPairsPerRow;
        if (r >= rows) continue;
        const int32_t t = qrow0 + r;
        const int32_t b = t / per_seq;
        const int32_t sq = t - (t / a.dec_Sq) * a.dec_Sq;
        if (!in_bounds(t >= 0 && b >= 0 && b < a.B && r < kBlockM && 8 * c + 8 <= kHalf)) continue;
        const float* inv = a.dec_inv ? a.dec_inv + static_cast<int64_t>(b) * kHalf : a.dec_inv_host;
        float sn[8], cs[8];
        sincos8(static_cast<float>(__ldg(a.dec_qpos + static_cast<int64_t>(b) * a.dec_Sq + sq)), inv + 8 * c, sn, cs);
        uint32_t pr[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            __half2 hc = __floats2half2_rn(cs[2 * k], cs[2 * k + 1]);
            __half2 hs = __floats2half2_rn(sn[2 * k], sn[2 * k + 1]);
            pr[2 * k] = *reinterpret_cast<uint32_t*>(&hc);
            pr[2 * k + 1] = *reinterpret_cast<uint32_t*>(&hs);
        }
        // 16-byte chunk positions of frequencies 8c..8c+3 and 8c+4..8c+7 in a table row, each
        // in its 128-byte box (atom), chunk index swizzled by the row
        const int p0 = (kHalf == 64) ? c : 2 * c;
        const int p1 = (kHalf == 64) ? 8 + c : 2 * c + 1;
        auto at = [&](int pc) -> uint32_t {
            return tab + static_cast<uint32_t>(pc >> 3) * AttnCfg<D>::kAtomBytes + static_cast<uint32_t>(r) * 128u +
                   ((static_cast<uint32_t>(pc & 7) ^ static_cast<uint32_t>(r & 7)) << 4);
        };
        sts128(at(p0), make_uint4(pr[0], pr[1], pr[2], pr[3]));
        sts128(at(p1), make_uint4(pr[4], pr[5], pr[6], pr[7]));
    }
}

// Angles of one RoPE thread for a key tile whose rows hold consecutive
// positions: 4 groups of 2 frequencies, (cos, sin) kept as packed fp32 pairs.
struct RecState {
    uint64_t c[4], s[4];     // current row's (cos f0, cos f1), (sin f0, sin f1)
};
// (c, s) <- (c, s) * (wc, ws) as complex numbers, two frequencies at a time;
// nws = -ws, so each part is one multiply and one fused multiply-add.
__device__ __forceinline__ void rec_step(uint64_t& c, uint64_t& s, uint64_t wc, uint64_t ws, uint64_t nws) {
    const uint64_t cn = ffma2(c, wc, fmul2(s, nws));
    s = ffma2(s, wc, fmul2(c, ws));
    c = cn;
}
__device__ __forceinline__ uint64_t fneg2(uint64_t v) { return v ^ 0x8000000080000000ull; }

// Rotate one task's two chunks with the angles of `e` (4 packed pairs of
// frequencies 8cp .. 8cp+7).
template <bool kFP16, bool kAdj>
__device__ __forceinline__ void rotate8_state(uint4& x1, uint4& x2, const RecState& e) {
    uint32_t* xa = reinterpret_cast<uint32_t*>(&x1);
    uint32_t* xb = reinterpret_cast<uint32_t*>(&x2);
    if constexpr (kAdj) {
        // word k of x1 is pair 8cp + k, of x2 pair 8cp + 4 + k: words (2m, 2m + 1) take the
        // packed angles of frequencies 8cp + 2m, + 1 (x2: 8cp + 4 + 2m, + 1)
        rot_adj2<kFP16>(xa[0], xa[1], e.c[0], e.s[0]);
        rot_adj2<kFP16>(xa[2], xa[3], e.c[1], e.s[1]);
        rot_adj2<kFP16>(xb[0], xb[1], e.c[2], e.s[2]);
        rot_adj2<kFP16>(xb[2], xb[3], e.c[3], e.s[3]);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint64_t X1 = IoT<kFP16>::unpack2(xa[k]);
            const uint64_t X2 = IoT<kFP16>::unpack2(xb[k]);
            xa[k] = pack2<kFP16>(fsub2(fmul2(X1, e.c[k]), fmul2(X2, e.s[k])));  // x1 cos - x2 sin
            xb[k] = pack2<kFP16>(ffma2(X2, e.c[k], fmul2(X1, e.s[k])));        // x2 cos + x1 sin
        }
    }
}

// Rotate a tile whose rows hold consecutive positions, without a table.
// This thread's rows are r0, r0 + step, ...; z holds the angles of row r0 and
// (wc, ws) advance them by `step` rows.  On return z holds the angles of row
// r0 + 128, the same thread's first row of the next tile.
template <int D, bool kFP16, bool kAdj, int kThreads = kRopeThreads>
__device__ __forceinline__ void rope_tile_rec(uint32_t tile, int32_t rows, int32_t rt, RecState& z,
                                              const uint64_t (&wc)[4], const uint64_t (&ws)[4]) {
    constexpr int kPairsPerRow = D / 16;
    constexpr int kIters = kBlockM * kPairsPerRow / kThreads;
    constexpr int kStep = kThreads / kPairsPerRow;
    const int cp = rt % kPairsPerRow;
    const int r0 = rt / kPairsPerRow;
    // This thread's rows are kStep apart, a multiple of the 8-row swizzle period, so every row's
    // chunks sit at row r0's offsets plus a multiple of kStep * 128 bytes.
    static_assert(kStep % 8 == 0, "rows of a thread share the swizzle pattern");
    uint32_t o1, o2;
    task_chunks<D, kAdj>(tile, r0, cp, o1, o2);
    // Unrolled by 4 (a key tile's 8 rows per thread in two passes; a query tile's 4 in one):
    // measured +0.4-1.2 % over 2 and -3 % with 1 on the prefill workloads, while a full unroll
    // (8) spills more and lost 0.5-3 %.
#pragma unroll 4
    for (int it = 0; it < kIters; ++it) {
        const int r = r0 + it * kStep;
        if (r < rows && task_in_tile<D>(r, cp)) {
            const uint32_t d = static_cast<uint32_t>(it * kStep * 128);
            uint4 x1 = lds128(o1 + d), x2 = lds128(o2 + d);
            rotate8_state<kFP16, kAdj>(x1, x2, z);
            sts128(o1 + d, x1);
            sts128(o2 + d, x2);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) rec_step(z.c[k], z.s[k], wc[k], ws[k], fneg2(ws[k]));
    }
}

// Recurrence state of RoPE thread rt for row r0 = rt / (D/16) of a sequence's
// first tile (angles (P + r0) w for its 8 frequencies), and the step (wc, ws)
// of kStep rows, both from the sequence's seeds.
// Angles of row `row` (relative to the sequence's first position P) for the
// 8 frequencies w[0..7] of a RoPE thread: the angle (P + row) w is formed in
// fp64 (exact for the fp32 w and any int32 P), reduced modulo 2 pi in fp64,
// and its cos/sin taken on the SFU -- the seeds' method, so a query tile's
// first rows are as accurate as the key tiles' seeds.
__device__ __forceinline__ void angles_at(int32_t P, int32_t row, const float (&w)[8], RecState& z) {
    const double two_pi = 6.283185307179586476925286766559;
    const double inv_two_pi = 0.15915494309189533576888376337251;
    const double p = static_cast<double>(P) + static_cast<double>(row);
    float c[8], sn[8];
#pragma unroll
    for (int f = 0; f < 8; ++f) {
        const double a = p * static_cast<double>(w[f]);
        const double r = fma(-two_pi, rint(a * inv_two_pi), a);
        __sincosf(static_cast<float>(r), &sn[f], &c[f]);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        z.c[k] = f2pack(c[2 * k], c[2 * k + 1]);
        z.s[k] = f2pack(sn[2 * k], sn[2 * k + 1]);
    }
}

// Rotate the first `rows` rows of a tile with cos/sin rows read from the
// global table (tab points at the tile's first row; D/2 32-bit words per row,
// laid out as rope_table_kernel writes them), by kThreads threads (tid <
// kThreads).  The table loads of kBatch rows are issued together, so one round
// trip to L2 covers each batch.
template <int D, bool kFP16, bool kAdj, int kThreads, int kBatch = 2>
__device__ __forceinline__ void rope_tile_global(uint32_t tile, const uint32_t* tab, int32_t rows, int32_t tid) {
    constexpr int kPairsPerRow = D / 16;
    constexpr int kIters = kBlockM * kPairsPerRow / kThreads;
    constexpr int kStep = kThreads / kPairsPerRow;
    const int cp = tid % kPairsPerRow;
    const int r0 = tid / kPairsPerRow;
    // chunk positions of the task's two frequency groups within a row, in the order its chunks
    // are taken (8cp..8cp+3 then 8cp+4..8cp+7, the other way round for a swapped task)
    const bool swp = task_swapped<D, kAdj>(cp);
    const int g0 = (D == 128) ? (swp ? 8 + cp : cp) : 2 * cp;
    const int g1 = (D == 128) ? (swp ? cp : 8 + cp) : 2 * cp + 1;
    if (!task_in_tile<D>(r0, cp) || !in_bounds(g0 < D / 8 && g1 < D / 8)) return;
#pragma unroll 1
    for (int b0 = 0; b0 < kIters; b0 += kBatch) {
        uint4 t0[kBatch], t1[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int r = r0 + (b0 + u) * kStep;
            if (b0 + u < kIters && r < rows) {
                const uint4* row = reinterpret_cast<const uint4*>(tab + static_cast<int64_t>(r) * (D / 2));
                t0[u] = __ldg(row + g0);
                t1[u] = __ldg(row + g1);
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int r = r0 + (b0 + u) * kStep;
            if (b0 + u >= kIters || r >= rows) break;
            uint32_t o1, o2;
            task_chunks<D, kAdj>(tile, r, cp, o1, o2);
            uint4 x1 = lds128(o1), x2 = lds128(o2);
            if constexpr (kAdj)
                rotate8_adj<kFP16>(x1, x2, t0[u], t1[u]);
            else
                rotate8<kFP16>(x1, x2, t0[u], t1[u]);
            sts128(o1, x1);
            sts128(o2, x2);
        }
    }
}

// 2^d for an integer-valued d <= 0 (or -inf), exactly: 0 below 2^-126.
__device__ __forceinline__ float exp2_int(float d) {
    return d < -126.0f ? 0.0f : __int_as_float((static_cast<int32_t>(d) + 127) << 23);
}
// Multiply 16 words of packed P (two bf16/fp16 values each) by f, a power of
// two (exact but for underflow).
template <bool kFP16>
__device__ __forceinline__ void scale_p(uint32_t (&w)[16], float f) {
    const uint64_t f2 = f2pack(f, f);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const float2 v = IoT<kFP16>::unpack(w[e]);
        w[e] = pack2<kFP16>(fmul2(f2pack(v.x, v.y), f2));
    }
}

// Columns c >= lim of a 32-column slice of S are masked (-inf).
__device__ __forceinline__ void mask_cols(uint32_t (&sr)[32], int32_t lim) {
    if (lim < 32) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
            if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
    }
}

// Bounded wait that ignores the abort flag: used to drain in-flight async
// copies and MMAs before the CTA exits.
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_status(5 /* RFA_ERR_TIMEOUT */);
            return;
        }
    }
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16, A = P in TMEM; only where `issue` is nonzero.
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate, uint32_t issue) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.ne.b32 e, %5, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(issue)
        : "memory");
}


// Key-tile counts of a work item: n0 / n1 key tiles read by query tile 0 / 1
// (0: tile absent), n_kv key tiles loaded.  Decode has one query tile and two
// independent chains over alternate key tiles: tile j goes to S/O buffer
// j % 2, and the two buffers' results are merged before the store.
struct ItemShape {
    int32_t nq, n0, n1, n_kv;
};
// One slot of the item ring in shared memory: the index (-1: none left, -2:
// the producer gave up) and, for an index >= 0, the item decoded once by the
// producer for all readers.
struct ItemSlot {
    int32_t x;
    WorkItem w;
    ItemShape sh;
};
static_assert(2 * sizeof(ItemSlot) <= 128, "item ring slots");

template <bool kDecode>
__device__ __forceinline__ ItemShape item_shape(const AttnArgs& a, const WorkItem& w) {
    ItemShape sh;
    sh.nq = (w.qt[1] >= 0) ? 2 : 1;
    const int32_t nkt = (w.L + kBlockN - 1) / kBlockN;
    sh.n0 = kDecode ? (nkt + 1) / 2 : (a.causal ? (w.qt[0] + 1) : nkt);
    sh.n1 = kDecode ? nkt / 2 : ((sh.nq == 1) ? 0 : (a.causal ? (w.qt[1] + 1) : nkt));
    sh.n_kv = kDecode ? nkt : max(sh.n0, sh.n1);
    return sh;
}

// Persistent: one CTA per SM takes work items one after another from a shared
// counter (decode: one CTA per item).  The Q/K producer fetches the item
// indices and passes them to the other roles through a two-slot ring in
// shared memory; every barrier phase runs on across items, so the next item's
// key tiles and query tiles load (and rotate) while the current item's last
// tiles are still in the softmax and the tensor pipe.
template <int D, bool kFP16, bool kAdj, bool kDecode>
__global__ void __launch_bounds__(kAttnThreads, 1)
    fused_rope_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmT,
                               const __grid_constant__ CUtensorMap tmO, const __grid_constant__ AttnArgs a) {
    using C = AttnCfg<D>;
    static_assert(C::kTabBytes <= C::kTileBytes, "decode stages the queries' cos/sin rows in a query slot");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    if ((sbase & 1023u) != 0u) {  // 128B-swizzled TMA/UMMA tiles need 1024-byte alignment
        if (threadIdx.x == 0) record_status(2 /* RFA_ERR_UNSUPPORTED */);
        return;
    }
    uint8_t* smem = smem_raw;
    volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + C::kOffAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffTmemSlot);
    ItemSlot* item_slot = reinterpret_cast<ItemSlot*>(smem + C::kOffItem);
    auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8u * static_cast<uint32_t>(i); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if constexpr (kDecode) {
        // the combine kernel that follows may place its blocks (they wait for this grid) as soon
        // as every decode block has started
        griddep_launch_dependents();
        const WorkItem w = decode_item_kv(a, blockIdx.x);
        if (threadIdx.x == 0 && w.split == 0) {
            const int32_t len = a.kv_lens[w.seq];
            if (len < a.dec_Sq || len > a.dec_max_len) record_status(1 /* RFA_ERR_INVALID_ARG */);
        }
        if (w.L <= 0) {
            // no keys in this split (past the sequence's length): an empty partial, or, with
            // one split, zero rows; the CTA returns before any barrier or TMEM is set up
            const int32_t rq = a.Hq * a.dec_Sq * a.B;
            for (int r = threadIdx.x; r < a.G * a.dec_Sq; r += blockDim.x) {
                if (a.dec_splits > 1) {
                    const int64_t pr = static_cast<int64_t>(w.split) * rq + w.qrow0 + r;
                    if (!in_bounds(pr >= 0 && pr < static_cast<int64_t>(a.dec_splits) * rq)) continue;
                    a.part_ml[2 * pr] = -INFINITY;
                    a.part_ml[2 * pr + 1] = 0.0f;
                } else {
                    const int64_t o = static_cast<int64_t>(w.qrow0 + r) * D;
                    if (!in_bounds(o >= 0 && o + D <= a.out_elems)) continue;
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + o);
                    for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            return;
        }
    }

    // consumer warps of the item ring: 16 softmax, 4 RoPE, the MMA and the V producer warp
    constexpr uint32_t kItemReaders = kSoftmaxWarps + kRopeWarps + 2;
    if (threadIdx.x == 0) {
        mbar_init(bar(C::kBarQFull), 1);
        mbar_init(bar(C::kBarQReady + 0), kDecode ? kRopeWarps : 8);
        mbar_init(bar(C::kBarQReady + 1), 8);
        mbar_init(bar(C::kBarQEmpty), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(C::kBarItemFull + s), 1);
            mbar_init(bar(C::kBarItemEmpty + s), kItemReaders);
        }
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(bar(C::kBarKFull + s), 1);
            mbar_init(bar(C::kBarVFull + s), 1);
            mbar_init(bar(C::kBarKReady + s), kRopeWarps);
            mbar_init(bar(C::kBarKEmpty + s), 1);
            mbar_init(bar(C::kBarVEmpty + s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(C::kBarSFull + i), 1);
            mbar_init(bar(C::kBarPFull + i), 8);  // one arrival per softmax warp of query tile i
            mbar_init(bar(C::kBarOFull + i), 1);
        }
        mbar_init(bar(C::kBarMmaFin), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Prefill, D = 128, with every sequence's positions consecutive (the flag the seed and table
    // kernels leave in the workspace) and an output tensor map: whole output tiles are staged in the
    // then unused cos/sin slot and written by TMA, which keeps the row-per-thread stores (32 rows
    // 256 bytes apart per instruction) off the SM's load/store path at item boundaries.
    const bool tstore = !kDecode && D == 128 && a.tma_out != 0 && a.sched != nullptr &&
                        *static_cast<const volatile int32_t*>(a.sched + 2) != 0;

    // The k-th item index of this CTA, -1 when none is left: decode serves
    // blockIdx.x alone; otherwise the shared counter hands out items in order
    // (longest first within the work order, see decode_item).
    auto fetch = [&](int32_t k) -> int32_t {
        if constexpr (kDecode) {
            return k == 0 ? static_cast<int32_t>(blockIdx.x) : -1;
        } else {
            if (!in_bounds(a.sched != nullptr)) return -1;
            const int32_t x = atomicAdd(a.sched, 1);
            return x < a.n_items ? x : -1;
        }
    };
    // Consumer side of the ring: wait for the k-th slot (nullptr if the wait gave up), read
    // what the role needs from it, then release it.  Called by lane 0 alone (warp_wide false)
    // or by all lanes of a warp, which then all read the slot before lane 0 releases it.
    auto wait_item = [&](int32_t k) -> const ItemSlot* {
        const int s = k & 1;
        // the wait's acquire orders the slot reads after the producer's writes
        return mbar_wait(bar(C::kBarItemFull + s), static_cast<uint32_t>(k >> 1) & 1u, abort_flag) ? item_slot + s
                                                                                                  : nullptr;
    };
    auto release_item = [&](int32_t k, bool warp_wide) {
        if (warp_wide) __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::kBarItemEmpty + (k & 1)));
    };
    auto read_item = [&](int32_t k, bool warp_wide, WorkItem& w, ItemShape& sh) -> int32_t {
        const ItemSlot* sl = wait_item(k);
        int32_t x = -2;
        if (sl != nullptr) {
            x = sl->x;
            w = sl->w;
            sh = sl->sh;
        }
        release_item(k, warp_wide);
        return x;
    };
    auto item_of = [&](int32_t x) -> WorkItem {
        in_bounds(x >= 0 && x < a.n_items);
        const WorkItem w = kDecode ? decode_item_kv(a, x) : decode_item(a, x);
        item_in_bounds(a, w, kDecode);
        return w;
    };
    // consecutive positions: K (and Q) angles come from the recurrence, no cos/sin rows per
    // K tile (decode: the cached keys are already rotated)
    auto consecutive = [&](const WorkItem& w) -> bool {
        return !kDecode && in_bounds(w.orig >= 0 && w.orig < a.B) && a.seeds[w.orig].consecutive != 0;
    };

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ Q/K producer (+ item fetch)
        // Both producer warps run converged, their waits voted across the lanes; lane 0 alone
        // fetches, writes the item slots, arrives and issues the copies (a single-lane branch
        // around the whole loop is starved of issue slots by the busy warps beside it).
        {
            const uint32_t leader = (lane == 0) ? 1u : 0u;
            auto wait = [&](uint32_t b, uint32_t parity) {
                return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag));
            };
            if (leader) {
                tma_prefetch_desc(&tmQ);
                tma_prefetch_desc(&tmK);
                tma_prefetch_desc(&tmT);
            }
            auto fetch_all = [&](int32_t k) -> int32_t {
                int32_t x = 0;
                if (leader) x = fetch(k);
                return __shfl_sync(0xffffffffu, x, 0);
            };
            auto publish = [&](int32_t k, int32_t x) -> bool {
                const int s = k & 1;
                if (k >= 2 && !wait(bar(C::kBarItemEmpty + s), static_cast<uint32_t>((k >> 1) - 1) & 1u))
                    return false;
                if (leader) {
                    item_slot[s].x = x;
                    if (x >= 0) {
                        const WorkItem w = item_of(x);
                        item_slot[s].w = w;
                        item_slot[s].sh = item_shape<kDecode>(a, w);
                    }
                    mbar_arrive(bar(C::kBarItemFull + s));  // release: the slot's contents are visible to the waiters
                }
                __syncwarp();  // the other lanes read the slot back
                return true;
            };
            const bool bnsd = (a.layout == 0);
            uint32_t g = 0;        // key tiles issued so far (ring position)
            int32_t q_items = 0;   // items whose query tiles were issued
            int32_t cur = fetch_all(0);
            // held: no item is published; the readers' item waits run out, this warp only drains
            bool ok = *static_cast<volatile int32_t*>(&g_hold_items) == 0 && publish(0, cur);
            for (int32_t it = 0; ok && cur >= 0; ++it) {
                const int32_t nxt = fetch_all(it + 1);
                if (!publish(it + 1, nxt)) break;
                const WorkItem w = item_slot[it & 1].w;  // published by this thread for item it
                const ItemShape sh = item_slot[it & 1].sh;
                const int32_t kvplane = bnsd ? (w.seq * a.Hkv + w.kvh) : w.kvh;
                const bool ktab = !kDecode && !consecutive(w);  // cos/sin rows staged beside each K tile
                const uint32_t kbytes = C::kTileBytes + (ktab ? C::kTabBytes : 0);
                auto load_tile = [&](const CUtensorMap* m, uint32_t dst, uint32_t b, int32_t plane, int32_t row0) {
                    // the copy engine clips boxes outside the tensor itself: record, then issue anyway
                    in_bounds(row0 >= 0 && row0 < w.L && plane >= 0 &&
                              (bnsd ? (plane < a.B * (m == &tmQ ? a.Hq : a.Hkv))
                                    : (plane < (m == &tmQ ? a.Hq : a.Hkv))));
                    for (int at = 0; at < C::kAtoms; ++at) {
                        if (bnsd)
                            tma_load_3d(dst + at * C::kAtomBytes, m, b, at * 64, row0, plane, leader);
                        else
                            tma_load_3d(dst + at * C::kAtomBytes, m, b, at * 64, plane, w.tok0 + row0, leader);
                    }
                };
                auto load_k = [&](int32_t j) -> bool {
                    const int s = g % C::kStages;
                    const uint32_t u = g / C::kStages;
                    if (u > 0 && !wait(bar(C::kBarKEmpty + s), (u - 1) & 1u)) return false;
                    if (ktab && g >= static_cast<uint32_t>(C::kTStages)) {
                        // the rows slot held the rows of key tile g - kTStages: wait until that tile is rotated
                        const uint32_t gp = g - C::kTStages;
                        if (!wait(bar(C::kBarKReady + gp % C::kStages), (gp / C::kStages) & 1u))
                            return false;
                    }
                    mbar_expect_tx(bar(C::kBarKFull + s), kbytes, leader);
                    load_tile(&tmK, sbase + C::kOffK + s * C::kTileBytes, bar(C::kBarKFull + s), kvplane, j * kBlockN);
                    if (ktab) {
                        const uint32_t dst = sbase + C::kOffT + (g % C::kTStages) * C::kTabBytes;
                        for (int bx = 0; bx < C::kTabBoxes; ++bx)
                            tma_load_3d(dst + bx * C::kAtomBytes, &tmT, bar(C::kBarKFull + s), bx * 32,
                                        w.tok0 + j * kBlockN, 0, leader);
                    }
                    ++g;
                    return true;
                };
                // key tile 0 first (its slot frees before the query slots do), then the query tiles
                if (!load_k(0)) break;
                if (it > 0 && !wait(bar(C::kBarQEmpty), static_cast<uint32_t>(it - 1) & 1u)) break;
                mbar_expect_tx(bar(C::kBarQFull), static_cast<uint32_t>(sh.nq) * C::kTileBytes, leader);
                for (int i = 0; i < sh.nq; ++i) {
                    if constexpr (kDecode) {  // q viewed as [B*Hq*Sq, D]: the group's rows from qrow0
                        for (int at = 0; at < C::kAtoms; ++at)
                            tma_load_3d(sbase + C::kOffQ + at * C::kAtomBytes, &tmQ, bar(C::kBarQFull), at * 64, 0,
                                        w.qrow0, leader);
                    } else {
                        const int32_t qplane = bnsd ? (w.seq * a.Hq + w.h[i]) : w.h[i];
                        load_tile(&tmQ, sbase + C::kOffQ + i * C::kTileBytes, bar(C::kBarQFull), qplane,
                                  w.qt[i] * kBlockM);
                    }
                }
                q_items = it + 1;
                bool kok = true;
                for (int32_t j = 1; j < sh.n_kv && kok; ++j) kok = load_k(j);
                if (!kok) break;
                cur = nxt;
            }
            // Drain: every issued copy must have landed before the CTA exits (earlier phases
            // completed before their slots were reissued).
            if (q_items > 0) mbar_wait_drain(bar(C::kBarQFull), static_cast<uint32_t>(q_items - 1) & 1u);
            for (uint32_t t = (g > static_cast<uint32_t>(C::kStages) ? g - C::kStages : 0u); t < g; ++t)
                mbar_wait_drain(bar(C::kBarKFull + t % C::kStages), (t / C::kStages) & 1u);
        }
    } else if (warp == kTmaVWarp) {
        // ------------------------------------------------------------ V producer
        // converged like the Q/K producer: lane 0 takes the item and issues
        {
            const uint32_t leader = (lane == 0) ? 1u : 0u;
            if (leader) tma_prefetch_desc(&tmV);
            const bool bnsd = (a.layout == 0);
            uint32_t g = 0;  // value tiles issued so far
            bool ok = true;
            for (int32_t it = 0; ok; ++it) {
                int32_t x = -2, kvplane = 0, tok0 = 0, n_kv = 0;
                if (leader) {
                    WorkItem w;
                    ItemShape sh;
                    x = read_item(it, false, w, sh);
                    if (x >= 0) {
                        kvplane = bnsd ? (w.seq * a.Hkv + w.kvh) : w.kvh;
                        tok0 = w.tok0;
                        n_kv = sh.n_kv;
                    }
                }
                __syncwarp();
                x = __shfl_sync(0xffffffffu, x, 0);
                if (x < 0) break;
                kvplane = __shfl_sync(0xffffffffu, kvplane, 0);
                tok0 = __shfl_sync(0xffffffffu, tok0, 0);
                n_kv = __shfl_sync(0xffffffffu, n_kv, 0);
                for (int32_t j = 0; j < n_kv; ++j) {
                    const int s = g % C::kStages;
                    const uint32_t u = g / C::kStages;
                    if (u > 0 && !__all_sync(0xffffffffu, mbar_wait(bar(C::kBarVEmpty + s), (u - 1) & 1u, abort_flag))) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(bar(C::kBarVFull + s), C::kTileBytes, leader);
                    const uint32_t dst = sbase + C::kOffV + s * C::kTileBytes;
                    for (int at = 0; at < C::kAtoms; ++at) {
                        if (bnsd)
                            tma_load_3d(dst + at * C::kAtomBytes, &tmV, bar(C::kBarVFull + s), at * 64, j * kBlockN,
                                        kvplane, leader);
                        else
                            tma_load_3d(dst + at * C::kAtomBytes, &tmV, bar(C::kBarVFull + s), at * 64, kvplane,
                                        tok0 + j * kBlockN, leader);
                    }
                    ++g;
                }
            }
            for (uint32_t t = (g > static_cast<uint32_t>(C::kStages) ? g - C::kStages : 0u); t < g; ++t)
                mbar_wait_drain(bar(C::kBarVFull + t % C::kStages), (t / C::kStages) & 1u);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ tcgen05 issuer
        // The whole warp runs the loop, converged (every wait's outcome is voted across the
        // lanes); the elected lane issues the MMAs and commits.
        {
            const uint32_t leader = elect_one();
            auto wait = [&](uint32_t b, uint32_t parity) {
                return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag));
            };
            constexpr uint32_t kIdescQK = idesc_f16(IoT<kFP16>::kFmt, 0, 0, kBlockM, kBlockN);
            constexpr uint32_t kIdescPV = idesc_f16(IoT<kFP16>::kFmt, 0, 1, kBlockM, D);
            // S_i = Q_i' K'^T into TMEM buffer i (A = Q_i' and B = K' from shared memory), key tile
            // at ring position t.  The issuing thread must keep up with the tensor pipe (one
            // 128x128x16 MMA per ~64 cycles): a tile's descriptors are built once and each k-step
            // adds its byte offset >> 4 to the start-address field (shared addresses < 256 KB: no
            // carry out of it).
            auto issue_qk = [&](int i, uint32_t t) {
                const uint64_t kd = smem_desc_sw128(sbase + C::kOffK + (t % C::kStages) * C::kTileBytes, 16, 1024);
                const uint64_t qd = smem_desc_sw128(sbase + C::kOffQ + (kDecode ? 0 : i) * C::kTileBytes, 16, 1024);
                const uint32_t dS = tmem + C::kColS + i * kBlockN;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t koff16 = ((k >> 2) * C::kAtomBytes + (k & 3) * 32) >> 4;
                    umma_ss(dS, qd + koff16, kd + koff16, kIdescQK, k > 0 ? 1u : 0u, leader);
                }
                tc_commit(bar(C::kBarSFull + i), leader);
            };
            // O_i += P_i V (A = P_i from TMEM buffer i: keys [64h, 64h + 64) at columns [64h, 64h + 32);
            // B = the value tile at ring position t) (acc: O_i already holds a partial sum)
            auto issue_pv = [&](int i, uint32_t t, bool acc) {
                const uint64_t vd =
                    smem_desc_sw128(sbase + C::kOffV + (t % C::kStages) * C::kTileBytes, C::kAtomBytes, 1024);
                const uint32_t dO = tmem + C::kColO + i * D, aP = tmem + C::kColS + i * kBlockN;
#pragma unroll
                for (int k = 0; k < kBlockN / 16; ++k)
                    umma_ts(dO, aP + (k >> 2) * 64 + (k & 3) * 8, vd + ((k * 16 * 128) >> 4), kIdescPV,
                            (acc || k > 0) ? 1u : 0u, leader);
            };
            auto kready = [&](uint32_t t) {
                return wait(bar(C::kBarKReady + t % C::kStages), (t / C::kStages) & 1u);
            };
            uint32_t g = 0;                  // key/value tiles consumed so far (ring position)
            uint32_t pc[2] = {0u, 0u};       // PFull_i phases consumed so far
            bool ok = true;
            for (int32_t it = 0; ok; ++it) {
                // lane 0 takes the item from the ring; the warp follows its copy of the shape
                int32_t x = -2, n0 = 0, n1 = 0, n_kv = 0;
                if (lane == 0) {
                    WorkItem w;
                    ItemShape sh;
                    x = read_item(it, false, w, sh);
                    if (x >= 0) {
                        n0 = sh.n0;
                        n1 = sh.n1;
                        n_kv = sh.n_kv;
                    }
                }
                __syncwarp();
                x = __shfl_sync(0xffffffffu, x, 0);
                n0 = __shfl_sync(0xffffffffu, n0, 0);
                n1 = __shfl_sync(0xffffffffu, n1, 0);
                n_kv = __shfl_sync(0xffffffffu, n_kv, 0);
                if (x < 0) break;
                const uint32_t qpar = static_cast<uint32_t>(it) & 1u;
                ok = wait(bar(C::kBarQReady + 0), qpar);
                if constexpr (kDecode) {
                    // Two chains over alternate key tiles (tile j into buffer j % 2).  QK_i of tile
                    // j + 2 reuses S_i: it is issued after PV_i of tile j, which read P_i, and MMAs
                    // from this thread execute in order.
                    for (int32_t j = 0; j < 2 && j < n_kv && ok; ++j) {
                        ok = kready(g + j);
                        if (!ok) break;
                        tc_fence_after();
                        issue_qk(j, g + j);
                        tc_commit(bar(C::kBarKEmpty + (g + j) % C::kStages), leader);
                    }
                    for (int32_t j = 0; j < n_kv && ok; ++j) {
                        const uint32_t t = g + j;
                        const int i = j & 1;
                        ok = wait(bar(C::kBarVFull + t % C::kStages), (t / C::kStages) & 1u) &&
                             wait(bar(C::kBarPFull + i), pc[i] & 1u);
                        if (!ok) break;
                        ++pc[i];
                        tc_fence_after();
                        issue_pv(i, t, j >= 2);
                        if (j + 2 >= n_kv) tc_commit(bar(C::kBarOFull + i), leader);  // last tile of buffer i
                        tc_commit(bar(C::kBarVEmpty + t % C::kStages), leader);
                        if (j + 2 < n_kv) {
                            ok = kready(t + 2);
                            if (!ok) break;
                            tc_fence_after();
                            issue_qk(i, t + 2);
                            tc_commit(bar(C::kBarKEmpty + (t + 2) % C::kStages), leader);
                        }
                    }
                    tc_commit(bar(C::kBarQEmpty), leader);
                } else {
                    // Order per key tile j: PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1).  The item's
                    // last QK is followed by a commit to QEmpty, so the producer can load the next
                    // item's query tiles while this item's last PVs run.
                    if (ok) ok = kready(g);
                    if (ok) {
                        tc_fence_after();
                        if (n0 > 0) issue_qk(0, g);
                        ok = wait(bar(C::kBarQReady + 1), qpar);  // both groups arrive every item
                    }
                    if (ok) {
                        tc_fence_after();
                        if (n1 > 0) issue_qk(1, g);
                        tc_commit(bar(C::kBarKEmpty + g % C::kStages), leader);
                        if (n_kv == 1) tc_commit(bar(C::kBarQEmpty), leader);
                    }
                    for (int32_t j = 0; j < n_kv && ok; ++j) {
                        const uint32_t t = g + j;
                        const int32_t jn = j + 1;
                        ok = wait(bar(C::kBarVFull + t % C::kStages), (t / C::kStages) & 1u);
                        if (!ok) break;
                        if (j < n0) {
                            ok = wait(bar(C::kBarPFull + 0), pc[0] & 1u);
                            if (!ok) break;
                            ++pc[0];
                            tc_fence_after();
                            issue_pv(0, t, j > 0);
                            if (j == n0 - 1) tc_commit(bar(C::kBarOFull + 0), leader);
                        }
                        if (jn < n_kv) {
                            ok = kready(t + 1);
                            if (!ok) break;
                            tc_fence_after();
                            if (jn < n0) issue_qk(0, t + 1);
                        }
                        if (j < n1) {
                            ok = wait(bar(C::kBarPFull + 1), pc[1] & 1u);
                            if (!ok) break;
                            ++pc[1];
                            tc_fence_after();
                            issue_pv(1, t, j > 0);
                            if (j == n1 - 1) tc_commit(bar(C::kBarOFull + 1), leader);
                        }
                        tc_commit(bar(C::kBarVEmpty + t % C::kStages), leader);
                        if (jn < n_kv) {
                            if (jn < n1) issue_qk(1, t + 1);
                            tc_commit(bar(C::kBarKEmpty + (t + 1) % C::kStages), leader);
                            if (jn == n_kv - 1) tc_commit(bar(C::kBarQEmpty), leader);
                        }
                    }
                }
                g += static_cast<uint32_t>(n_kv);
            }
            tc_commit(bar(C::kBarMmaFin), leader);
            mbar_wait_drain(bar(C::kBarMmaFin), 0);
        }
    } else if (warp >= kRopeWarp0 && warp < kRopeWarp0 + kRopeWarps) {
        // ------------------------------------------------------------ RoPE warpgroup
        // Per item, one loop over the key tiles to rotate (decode: the query tile, after key tile
        // 0; prefill query tiles are rotated by the softmax warps).  Consecutive positions: the
        // first-row angles of key tile 0 are formed directly (angles_at); every row after that
        // by the step of kStep rows (a thread's rows of a tile, then on into the next key tile);
        // otherwise cos/sin rows from the table, staged beside the key tile by TMA.
        const int32_t rt = threadIdx.x - kRopeWarp0 * 32;  // 0..127
        constexpr int kPairsPerRow = D / 16;
        const int r0 = rt / kPairsPerRow;                   // this thread's first row of a tile
        uint32_t g = 0;  // key tiles rotated so far (ring position)
        for (int32_t it = 0;; ++it) {
            WorkItem w;
            ItemShape sh;
            if (read_item(it, true, w, sh) < 0) break;
            if constexpr (kDecode) decode_query_table<D>(sbase + C::kOffQ + C::kTileBytes, a, w.qrow0, rt);
            const bool rec = consecutive(w);
            uint64_t wc[4], ws[4];  // in-tile step (cos, sin) of kStep rows, packed pairs
            RecState zk;            // key tiles: this thread's first row of the next tile (recurrence)
            if (rec) {
                // key tile 0's first-row angles formed directly from the sequence's first position and
                // this thread's frequencies; every later row by the step
                const RopeSeed* sd = a.seeds + w.orig;
                const int cpr = rt % kPairsPerRow;  // this thread's frequency groups, in task order
                const float4 u0 = *reinterpret_cast<const float4*>(sd->inv + task_freq<D, kAdj>(cpr, 0));
                const float4 u1 = *reinterpret_cast<const float4*>(sd->inv + task_freq<D, kAdj>(cpr, 1));
                const float qw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float4 v = *reinterpret_cast<const float4*>(sd->wstep + task_freq<D, kAdj>(cpr, k >> 1) +
                                                                      2 * (k & 1));  // pairs f, f + 1
                    wc[k] = f2pack(v.x, v.z);
                    ws[k] = f2pack(v.y, v.w);
                }
                angles_at(sd->pos0, r0, qw, zk);
            }
            bool ok = true;
            // decode: key tile 0, the query tile, then the other key tiles; otherwise key tiles
            // only (the softmax warps rotate the query tiles)
            const int32_t nqr = kDecode ? sh.nq : 0;
            const int32_t nrot = sh.n_kv + nqr;
#pragma unroll 1
            for (int32_t e = 0; e < nrot && ok; ++e) {
                const bool isq = e >= 1 && e <= nqr;
                const int qi = e - 1;                          // query tile (isq)
                const int32_t j = (e == 0) ? 0 : e - nqr;      // key tile (!isq)
                const uint32_t t = g + static_cast<uint32_t>(j);
                const int s = t % C::kStages;
                uint32_t tile;
                int32_t row0;
                if (isq) {
                    if (qi == 0) ok = mbar_wait(bar(C::kBarQFull), static_cast<uint32_t>(it) & 1u, abort_flag);
                    tile = sbase + C::kOffQ + qi * C::kTileBytes;
                    row0 = w.qt[qi] * kBlockM;
                } else {
                    ok = mbar_wait(bar(C::kBarKFull + s), (t / C::kStages) & 1u, abort_flag);
                    tile = sbase + C::kOffK + s * C::kTileBytes;
                    row0 = j * kBlockN;
                }
                if (!ok) break;
                const int32_t rows = min(kBlockM, w.L - row0);
                if constexpr (kDecode) {
                    // cached keys are already rotated; the query tile holds the group's G * Sq rows,
                    // their cos/sin rows in the second query slot (decode_query_table above)
                    if (isq) rope_tile<D, kFP16, kAdj>(tile, sbase + C::kOffQ + C::kTileBytes, a.G * a.dec_Sq, rt);
                } else if (rec) {
                    // key tile j > 0 continues from the state key tile j - 1 left (its rows step on by 128)
                    rope_tile_rec<D, kFP16, kAdj>(tile, rows, rt, zk, wc, ws);
                } else {
                    rope_tile<D, kFP16, kAdj>(tile, sbase + C::kOffT + (t % C::kTStages) * C::kTabBytes, rows, rt);
                }
                fence_proxy_async_smem();  // rotated tile written by the generic proxy, read by the tensor cores
                __syncwarp();
                if (lane == 0) {
                    if (!isq)
                        mbar_arrive(bar(C::kBarKReady + s));
                    else if (qi == sh.nq - 1)
                        mbar_arrive(bar(C::kBarQReady + 0));
                }
            }
            g += static_cast<uint32_t>(sh.n_kv);
            if (!ok) break;
        }
    } else if (warp < kSoftmaxWarps) {
        // ------------------------------------------------------------ softmax warps
        // Query tile i has 8 warps: warp w covers TMEM lanes (rows) 32 (w % 4) .. + 31 and key
        // columns [64 hf, 64 hf + 64) of every score tile, hf = (w / 4) % 2.  The two warps of a
        // row exchange half-row maxima (then row sums) through shared memory at named barrier
        // 1 + i (256 threads), executed exactly n_i + 2 times per item by every one of them: a
        // failed (timed-out) wait only turns the remaining work into no-ops, it never skips a
        // barrier.  The 8 warps of a group decide together, with a bar.red.and at the group's
        // barrier (decode: all 16 at named barrier 3, which its merge also uses), whether to take
        // the next item, so the warps that share a barrier always run the same items.  A slot
        // written at tile j + 1
        // was read at tile j before the reader arrived on PFull_i(j), which S_i(j + 1) waits
        // for, so one slot per row and half suffices.
        const int i = warp >> 3;             // query tile
        const int hf = (warp >> 2) & 1;      // key-column half
        const int row = ((warp & 3) << 5) + lane;  // 0..127 == TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t sc = tmem + lane_off + C::kColS + i * kBlockN + hf * 64;  // this half of S_i; P over [0, 32)
        constexpr int kOHalf = D / 2;                                           // O_i columns rescaled / stored
        const uint32_t oc = tmem + lane_off + C::kColO + i * D + hf * kOHalf;
        float* xch = reinterpret_cast<float*>(smem + C::kOffXchg) + i * 2 * kBlockM;  // [half][row]
        const uint32_t nb = 1u + static_cast<uint32_t>(i);
        const float sl2 = a.scale_log2;
        uint32_t cs = 0;  // SFull_i phases consumed so far
        uint32_t co = 0;  // OFull_i phases consumed so far
        for (int32_t it = 0;; ++it) {
            // only the fields this role uses are read from the slot
            int32_t x = -2, n0 = 0, n1 = 0, nq = 0, L = 0, tok0 = 0, qt_i = 0, h_i = 0, seq = 0, split = 0, qrow0 = 0;
            int32_t orig = 0;
            if (const ItemSlot* sl = wait_item(it)) {
                x = sl->x;
                n0 = sl->sh.n0;
                n1 = sl->sh.n1;
                nq = sl->sh.nq;
                L = sl->w.L;
                tok0 = sl->w.tok0;
                qt_i = sl->w.qt[i];
                h_i = sl->w.h[i];
                seq = sl->w.seq;
                orig = sl->w.orig;
                if constexpr (kDecode) {
                    split = sl->w.split;
                    qrow0 = sl->w.qrow0;
                }
            }
            release_item(it, true);
            // Decode: the 16 warps decide together whether to take the item, as their merge
            // barrier (3) spans both groups.  Prefill: each group decides alone (the groups share
            // no named barrier), after rotating its query tile, so that each warp starts its rows
            // of the rotation as soon as its own epilogue is done rather than the group's slowest.
            if constexpr (kDecode) {
                if (!named_bar_and(3u, kSoftmaxWarps * 32u, x >= 0 && *abort_flag == 0)) break;
            }
            if (!kDecode && x >= 0) {
                // This group rotates its own query tile (idle until its first score tile); both
                // groups arrive on their QReady every item.  Consecutive positions: each thread's
                // first-row angles are formed directly from the sequence's seed and its other rows
                // follow by the recurrence (step of 32 rows, the square of the seed's 16-row step);
                // otherwise cos/sin rows come from the global table.
                bool qok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarQFull), static_cast<uint32_t>(it) & 1u, abort_flag));
                if (qok && i < nq) {
                    const int32_t q0 = qt_i * kBlockM;
                    const int32_t rows = min(kBlockM, L - q0);
                    const int32_t qtid = ((warp & 7) << 5) + lane;
                    const uint32_t qtile = sbase + C::kOffQ + i * C::kTileBytes;
                    const bool rec = in_bounds(orig >= 0 && orig < a.B) && a.seeds[orig].consecutive != 0;
                    if (rec) {
                        constexpr int kPairsPerRow = D / 16;
                        const RopeSeed* sd = a.seeds + orig;
                        const int cpq = qtid % kPairsPerRow;  // frequency groups in task order
                        const float4 u0 = *reinterpret_cast<const float4*>(sd->inv + task_freq<D, kAdj>(cpq, 0));
                        const float4 u1 = *reinterpret_cast<const float4*>(sd->inv + task_freq<D, kAdj>(cpq, 1));
                        const float qw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                        uint64_t wc[4], ws[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float4 v = *reinterpret_cast<const float4*>(
                                sd->wstep + task_freq<D, kAdj>(cpq, k >> 1) + 2 * (k & 1));
                            wc[k] = f2pack(v.x, v.z);
                            ws[k] = f2pack(v.y, v.w);
                            uint64_t c = wc[k], sn = ws[k];
                            rec_step(c, sn, wc[k], ws[k], fneg2(ws[k]));  // twice the seed's step
                            wc[k] = c;
                            ws[k] = sn;
                        }
                        RecState zq;
                        angles_at(sd->pos0, q0 + qtid / kPairsPerRow, qw, zq);
                        rope_tile_rec<D, kFP16, kAdj, 256>(qtile, rows, qtid, zq, wc, ws);
                    } else if (in_bounds(q0 >= 0 && static_cast<int64_t>(tok0) + q0 + rows <= a.ntok)) {
                        rope_tile_global<D, kFP16, kAdj, 256>(qtile, a.table + static_cast<int64_t>(tok0 + q0) * (D / 2),
                                                              rows, qtid);
                    }
                    fence_proxy_async_smem();  // Q' written by the generic proxy, read by the tensor cores
                }
                __syncwarp();
                if (qok && lane == 0) mbar_arrive(bar(C::kBarQReady + i));
            }
            if constexpr (!kDecode) {
                if (!named_bar_and(nb, 256u, x >= 0 && *abort_flag == 0)) break;
            }
            const int32_t n_i = i == 0 ? n0 : n1;
            const int32_t qi = qt_i * kBlockM + row;
            int32_t vis = a.causal ? min(qi + 1, L) : L;  // keys [0, vis) visible to this row
            if constexpr (kDecode) {
                // row = g * Sq + s: new token s of the sequence's last Sq sees keys up to len - Sq + s
                // (bottom-right causal), relative to this split's first key
                const int32_t len = in_bounds(seq >= 0 && seq < a.B) ? min(max(a.kv_lens[seq], 0), a.dec_Smax) : 0;
                vis = a.causal ? min(L, len - a.dec_Sq + row % a.dec_Sq + 1 - split * a.dec_chunk) : L;
            }
            // prefill epilogue: this thread's output half-row (computed now, so the item's other
            // fields need not stay live through the tile loop)
            int64_t o_off = 0;
            bool o_valid = false;
            if constexpr (!kDecode) {
                o_valid = qi < L;
                o_off = (a.layout == 0) ? ((static_cast<int64_t>(seq) * a.Hq + h_i) * a.S + qi) * D
                                        : (static_cast<int64_t>(tok0 + qi) * a.Hq + h_i) * D;
                o_off += hf * kOHalf;
            }
            // m: the row's reference maximum of score * scale * log2(e), identical in both halves and
            // an integer (or -inf before the row's first visible key), so every rescale below is by
            // an exact power of two.  It may lag the true maximum by up to 2^kRescaleThreshold.
            float m = -INFINITY;
            float l = 0.0f;       // this half's running sum of exp2(score * scale_log2 - m)
            bool ok = true;       // warp-uniform; tcgen05.ld/st are warp-collective
            for (int32_t j = 0; j < n_i; ++j) {
                ok = ok && __all_sync(0xffffffffu, mbar_wait(bar(C::kBarSFull + i), cs & 1u, abort_flag));
                ++cs;
                const int32_t kt = kDecode ? 2 * j + i : j;          // key tile of this step
                const int32_t lim = vis - kt * kBlockN - hf * 64;  // columns [0, lim) of this half are visible
                // One read of this half of S, 32 columns at a time: a chunk's maximum is checked
                // against this half's reference mt and its exponentials taken in the same pass.  A
                // chunk more than 2^kRescaleThreshold above mt raises mt to the ceiling of its maximum,
                // and the chunk this tile already wrote owes the factor 2^(old - new).  P is written
                // over the half's S columns already read (P columns [16q, 16q + 16) lie in [0, 32q + 32)).
                float mt = m;     // this half's reference for this tile
                float lt = 0.0f;  // this half's sum of this tile's P (relative to mt)
                float f0 = 1.0f;  // factor owed by chunk 0's P after chunk 1 raised mt
                if (ok) {
                    tc_fence_after();
                    const uint64_t sl2x2 = f2pack(sl2, sl2);
#pragma unroll 1
                    for (int q = 0; q < 2; ++q) {
                        uint32_t sr[32];
                        tmem_ld32(sc + q * 32, sr);
                        tmem_wait_ld();
                        mask_cols(sr, lim - q * 32);
                        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                        for (int c = 0; c < 32; c += 2)
                            mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
                        const float cm = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * sl2;
                        if (cm > mt + kRescaleThreshold) {
                            const float mr = ceilf(cm);
                            const float f = exp2_int(mt - mr);
                            lt *= f;
                            if (q == 1) f0 = f;
                            mt = mr;
                        }
                        const float neg_m = (mt == -INFINITY) ? 0.0f : -mt;
                        const uint64_t negm2 = f2pack(neg_m, neg_m);
                        uint64_t l2[2] = {0ull, 0ull};  // packed (+0.0f, +0.0f)
#pragma unroll
                        for (int c2 = 0; c2 < 16; ++c2) {
                            const uint64_t sv = f2pack(__uint_as_float(sr[2 * c2]), __uint_as_float(sr[2 * c2 + 1]));
                            const float2 xv = f2unpack(ffma2(sv, sl2x2, negm2));
                            const uint64_t pp = f2pack(ex2(xv.x), ex2(xv.y));
                            l2[c2 & 1] = fadd2(l2[c2 & 1], pp);
                            sr[c2] = pack2<kFP16>(pp);
                        }
                        tmem_st16(sc + q * 16, reinterpret_cast<const uint32_t(&)[16]>(sr));
                        const float2 la = f2unpack(fadd2(l2[0], l2[1]));
                        lt += la.x + la.y;
                    }
                    if (__any_sync(0xffffffffu, f0 != 1.0f)) {
                        uint32_t pw[16];
                        tmem_ld16(sc, pw);
                        tmem_wait_ld();
                        scale_p<kFP16>(pw, f0);
                        tmem_st16(sc, pw);
                    }
                }
                // The two halves agree on the larger reference: a half below it rescales its P and its
                // tile sum; when the row's reference rose, O (which holds PV_i(j-1): issued before
                // QK_i(j), whose completion we saw) and the running sum follow.
                xch[hf * kBlockM + row] = mt;
                named_bar_sync(nb, 256);
                ok = __all_sync(0xffffffffu, ok && *abort_flag == 0);
                if (!ok) continue;
                const float mf = fmaxf(mt, xch[(hf ^ 1) * kBlockM + row]);
                if (__any_sync(0xffffffffu, mf != mt)) {
                    const float f = exp2_int(mt - mf);
                    lt *= f;
                    uint32_t pw[16];
#pragma unroll 1
                    for (int q = 0; q < 2; ++q) {
                        tmem_ld16(sc + q * 16, pw);
                        tmem_wait_ld();
                        scale_p<kFP16>(pw, f);
                        tmem_st16(sc + q * 16, pw);
                    }
                }
                const bool rise = mf > m;
                if (j > 0 && __any_sync(0xffffffffu, rise)) {
                    const float alpha = rise ? exp2_int(m - mf) : 1.0f;
                    const uint64_t alpha2 = f2pack(alpha, alpha);
                    l *= alpha;
#pragma unroll 1
                    for (int q = 0; q < kOHalf / 32; ++q) {
                        uint32_t o[32];
                        tmem_ld32(oc + q * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; c += 2) {
                            const float2 v = f2unpack(fmul2(f2pack(__uint_as_float(o[c]), __uint_as_float(o[c + 1])), alpha2));
                            o[c] = __float_as_uint(v.x);
                            o[c + 1] = __float_as_uint(v.y);
                        }
                        tmem_st32(oc + q * 32, o);
                    }
                }
                if (rise) m = mf;
                l += lt;
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::kBarPFull + i));
            }
            // epilogue: combine the two halves' row sums (the slot may still hold a maximum the
            // other half has yet to read, hence the barrier before writing), then out = O / l
            named_bar_sync(nb, 256);
            xch[hf * kBlockM + row] = l;
            named_bar_sync(nb, 256);
            l += xch[(hf ^ 1) * kBlockM + row];
            if constexpr (kDecode) {
                // The two buffers hold alternate key tiles of this split.  With M = max(m_0, m_1) and
                // c_b = 2^(m_b - M) (0 where l_b = 0): O = c_0 O_0 + c_1 O_1, l = c_0 l_0 + c_1 l_1.
                // Warp (i, hf) merges column quarter 2 i + hf of its lane group's rows.  (m, l) pass
                // through the K-tile cos/sin slot, which decode uses for nothing else: a buffer with
                // no tiles reaches this point while the query tile may still be in flight.  A decode
                // CTA runs one item, so both OFull phases are the first.
                float* mlx = reinterpret_cast<float*>(smem + C::kOffT);  // [m_0, m_1, l_0, l_1][row]
                if (hf == 0) {
                    mlx[i * kBlockM + row] = m;
                    mlx[(2 + i) * kBlockM + row] = l;
                }
                named_bar_sync(3, kSoftmaxWarps * 32);
                const float m0 = mlx[row], m1 = mlx[kBlockM + row];
                const float l0 = mlx[2 * kBlockM + row], l1 = mlx[3 * kBlockM + row];
                const bool fin = __all_sync(0xffffffffu, ok && *abort_flag == 0) &&
                                 __all_sync(0xffffffffu, mbar_wait(bar(C::kBarOFull + 0), 0, abort_flag)) &&
                                 (n1 == 0 || __all_sync(0xffffffffu, mbar_wait(bar(C::kBarOFull + 1), 0, abort_flag)));
                if (fin) {
                    tc_fence_after();
                    const float M = fmaxf(m0, m1);
                    const float c0 = (l0 > 0.0f) ? ex2(m0 - M) : 0.0f;
                    const float c1 = (l1 > 0.0f) ? ex2(m1 - M) : 0.0f;
                    const float lt = c0 * l0 + c1 * l1;
                    // rows of q viewed as [B*Hq*Sq, D]; with several splits, unnormalised fp32 O and
                    // (m, l) go to the partials that the combine kernel merges
                    bool valid = row < a.G * a.dec_Sq;
                    const bool partial = a.dec_splits > 1;
                    int64_t o_off = static_cast<int64_t>(qrow0 + row) * D;
                    if (partial) {
                        const int64_t rq = static_cast<int64_t>(a.B) * a.Hq * a.dec_Sq;
                        const int64_t pr = static_cast<int64_t>(split) * rq + qrow0 + row;
                        o_off = pr * D;
                        if (valid) valid = in_bounds(pr >= 0 && pr < a.dec_splits * rq);
                        if (valid && i == 0 && hf == 0) {
                            a.part_ml[2 * pr] = (lt > 0.0f) ? M : -INFINITY;
                            a.part_ml[2 * pr + 1] = lt;
                        }
                    }
                    if (valid && !partial) valid = in_bounds(o_off >= 0 && o_off + D <= a.out_elems);
                    const float scl = partial ? 1.0f : ((lt > 0.0f) ? 1.0f / lt : 0.0f);
                    const float w0 = c0 * scl, w1 = c1 * scl;
                    constexpr int kOQ = D / 4;  // columns per warp
                    const int c_lo = (2 * i + hf) * kOQ;
                    const uint32_t o0c = tmem + lane_off + C::kColO + c_lo;  // O_1 is D columns further
#pragma unroll 1
                    for (int q = 0; q < kOQ / 16; ++q) {
                        uint32_t o0[16], o1[16];
                        tmem_ld16(o0c + q * 16, o0);
                        if (n1 > 0) {
                            tmem_ld16(o0c + D + q * 16, o1);
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e) o1[e] = 0u;
                        }
                        tmem_wait_ld();
                        float v[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)  // a buffer with l = 0 contributes nothing (its O may be unset)
                            v[e] = (c0 > 0.0f ? w0 * __uint_as_float(o0[e]) : 0.0f) +
                                   (c1 > 0.0f ? w1 * __uint_as_float(o1[e]) : 0.0f);
                        if (!valid) continue;
                        if (partial) {
                            float4* dst = reinterpret_cast<float4*>(a.part_o + o_off + c_lo + q * 16);
#pragma unroll
                            for (int v4 = 0; v4 < 4; ++v4)
                                dst[v4] = make_float4(v[4 * v4], v[4 * v4 + 1], v[4 * v4 + 2], v[4 * v4 + 3]);
                        } else {
                            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + o_off + c_lo + q * 16);
#pragma unroll
                            for (int v4 = 0; v4 < 2; ++v4) {
                                uint32_t wv[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    wv[e] = pack2<kFP16>(f2pack(v[8 * v4 + 2 * e], v[8 * v4 + 2 * e + 1]));
                                dst[v4] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                            }
                        }
                    }
                }
            } else {
                bool fin = n_i > 0 && __all_sync(0xffffffffu, ok && *abort_flag == 0);
                if (n_i > 0) {
                    fin = fin && __all_sync(0xffffffffu, mbar_wait(bar(C::kBarOFull + i), co & 1u, abort_flag));
                    ++co;
                }
                bool staged = false;  // this group's tile went out through the staging slot
                if (tstore) {
                    // Group i stages in its own half of the slot, one 64-column swizzle atom at a
                    // time (the 4 warps of column half `at`, then TMA).  Whole tiles only: a tile
                    // that runs past its sequence would overwrite the next sequence's rows.
                    const int32_t q0 = qt_i * kBlockM;
                    staged = named_bar_and(nb, 256u, fin && q0 + kBlockM <= L);
                    if (staged) {
                        tc_fence_after();
                        const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
                        const uint64_t il2 = f2pack(inv_l, inv_l);
                        const uint32_t buf = sbase + C::kOffT + i * (C::kTabBytes / 2);
                        const uint32_t rbase = buf + row * 128;
#pragma unroll 1
                        for (int at = 0; at < 2; ++at) {
                            if (hf == at) {
                                // row `row`, 16-byte chunks 4q .. 4q + 3 at chunk ^ (row & 7)
#pragma unroll 1
                                for (int q = 0; q < kOHalf / 32; ++q) {
                                    uint32_t o[32];
                                    tmem_ld32(oc + q * 32, o);
                                    tmem_wait_ld();
                                    uint32_t wv[16];
#pragma unroll
                                    for (int e = 0; e < 16; ++e)
                                        wv[e] = pack2<kFP16>(
                                            fmul2(f2pack(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1])), il2));
#pragma unroll
                                    for (int c = 0; c < 4; ++c)
                                        sts128(rbase + (static_cast<uint32_t>((4 * q + c) ^ (row & 7)) << 4),
                                               make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]));
                                }
                                fence_proxy_async_smem();  // staged by the generic proxy, read by TMA
                            }
                            named_bar_sync(nb, 256);
                            if ((warp & 7) == 0 && lane == 0) {
                                if (a.layout == 0)
                                    tma_store_3d(&tmO, buf, at * 64, q0, seq * a.Hq + h_i);
                                else
                                    tma_store_3d(&tmO, buf, at * 64, h_i, tok0 + q0);
                                bulk_commit();
                                bulk_wait_read();  // the buffer may be staged again
                            }
                            named_bar_sync(nb, 256);
                        }
                    }
                }
                if (fin && !staged) {
                    tc_fence_after();
                    const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
                    bool valid = o_valid;
                    uint16_t* outp = reinterpret_cast<uint16_t*>(a.out);
                    if (valid) valid = in_bounds(o_off >= 0 && o_off + kOHalf <= a.out_elems);
                    const uint64_t il2 = f2pack(inv_l, inv_l);
                    // Each thread writes its row's kOHalf contiguous outputs: 32-byte stores (whole
                    // sectors) when the output is 32-byte aligned, else 16-byte ones.
                    const bool wide = (reinterpret_cast<uintptr_t>(a.out) & 31u) == 0;
#pragma unroll 1
                    for (int q = 0; q < kOHalf / 32; ++q) {
                        uint32_t o[32];
                        tmem_ld32(oc + q * 32, o);
                        tmem_wait_ld();
                        if (valid) {
                            uint32_t wv[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                wv[e] = pack2<kFP16>(fmul2(f2pack(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1])), il2));
                            uint16_t* dst = outp + o_off + q * 32;
                            if (wide) {
                                stg256(dst, reinterpret_cast<const uint32_t(&)[8]>(wv[0]));
                                stg256(dst + 16, reinterpret_cast<const uint32_t(&)[8]>(wv[8]));
                            } else {
                                uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                                for (int v4 = 0; v4 < 4; ++v4)
                                    d4[v4] = make_uint4(wv[4 * v4], wv[4 * v4 + 1], wv[4 * v4 + 2], wv[4 * v4 + 3]);
                            }
                        }
                    }
                }
                // the next item's PV_i(0) overwrites O_i only after this warp's PFull_i arrival of
                // that item, which follows these reads (tcgen05.wait::ld above)
            }
        }
        // staged tiles' stores complete before the CTA exits
        if (tstore && (warp & 7) == 0 && lane == 0) bulk_wait();
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
    if constexpr (!kDecode) {
        // The last CTA to finish re-zeroes the work counters for the next launch on this
        // workspace: every CTA counts itself in only after all its fetches (its producer is
        // done before the barrier above).
        if (threadIdx.x == 0) {
            __threadfence();
            if (atomicAdd(a.sched + 1, 1) == static_cast<int32_t>(gridDim.x) - 1) {
                atomicExch(a.sched, 0);
                atomicExch(a.sched + 1, 0);
                __threadfence();
            }
        }
    }
}

// Merge the split partials of decode attention: for every query row,
// out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s over the splits with
// l_s > 0 (M their largest m_s), rounded to bf16/fp16.  One thread per row and
// 8 consecutive columns.
template <bool kFP16>
__global__ void __launch_bounds__(256) decode_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_ml, void* out,
                                                             int32_t rows, int32_t D, int32_t splits) {
    griddep_wait();  // the decode grid's partials complete and visible (programmatic launch)
    const int32_t per_row = D / 8;
    const int64_t work = static_cast<int64_t>(rows) * per_row;
    for (int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; w < work;
         w += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int32_t r = static_cast<int32_t>(w / per_row);
        const int32_t c = static_cast<int32_t>(w - static_cast<int64_t>(r) * per_row) * 8;
        float M = -INFINITY;
        for (int32_t s = 0; s < splits; ++s) {
            const int64_t pr = static_cast<int64_t>(s) * rows + r;
            if (part_ml[2 * pr + 1] > 0.0f) M = fmaxf(M, part_ml[2 * pr]);
        }
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float den = 0.0f;
        for (int32_t s = 0; s < splits; ++s) {
            const int64_t pr = static_cast<int64_t>(s) * rows + r;
            const float ls = part_ml[2 * pr + 1];
            if (!(ls > 0.0f)) continue;
            const float wgt = exp2f(part_ml[2 * pr] - M);
            den = fmaf(wgt, ls, den);
            const float4* src = reinterpret_cast<const float4*>(part_o + pr * D + c);
            const float4 u = src[0], v = src[1];
            acc[0] = fmaf(wgt, u.x, acc[0]); acc[1] = fmaf(wgt, u.y, acc[1]);
            acc[2] = fmaf(wgt, u.z, acc[2]); acc[3] = fmaf(wgt, u.w, acc[3]);
            acc[4] = fmaf(wgt, v.x, acc[4]); acc[5] = fmaf(wgt, v.y, acc[5]);
            acc[6] = fmaf(wgt, v.z, acc[6]); acc[7] = fmaf(wgt, v.w, acc[7]);
        }
        const float inv = den > 0.0f ? 1.0f / den : 0.0f;
        if (!in_bounds(c + 8 <= D && static_cast<int64_t>(r) * D + c + 8 <= static_cast<int64_t>(rows) * D)) continue;
        uint32_t wv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) wv[e] = IoT<kFP16>::pack(acc[2 * e] * inv, acc[2 * e + 1] * inv);
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + static_cast<int64_t>(r) * D + c) =
            make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
}

}  // namespace rfa
