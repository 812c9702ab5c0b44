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
// One CTA = one work item (sequence, query head, 128-row query tile).  Warp roles:
//   warps 0-7  two softmax warpgroups; warpgroup g takes key columns
//              [64g, 64g + 64) of every score tile, thread t of it owns query
//              row t (TMEM lane t).  Per tile: load its half of S from TMEM,
//              mask, exchange the half-row maxima through shared memory (named
//              barrier 1 over the 256 softmax threads), keep
//              the running max (identical in both) and a partial sum, write P
//              (bf16/fp16) into TMEM, rescale its half of O only when the max
//              grows by > 2^8.  At the end the partial sums are combined and
//              each warpgroup normalises and stores half of the columns.
//   warps 8-11 RoPE warpgroup: rotates the Q tile once (then moves Q' into
//              TMEM, where the QK MMAs read it) and every K tile in place in
//              the 128B-swizzled shared-memory layout.  Element i and its
//              rotate-half partner i + D/2 sit at the same offset of two swizzle
//              atoms (D = 128) or in chunks c and c ^ 4 of one atom (D = 64).
//              K angles come from a complex recurrence in registers when the
//              sequence's positions are consecutive, else from cos/sin rows
//              that TMA staged next to the tile.
//   warp 12    TMA producer: Q (+ its cos/sin rows) once, then K tiles (+ rows
//              when needed) through a kStages ring.
//   warp 13    tcgen05 issuer (one thread) and TMEM owner: S_j = Q'K_j'^T into
//              TMEM buffer j % 2 (A = Q' from TMEM), O += P_j V_j (A = P from
//              TMEM, B = V from shared memory); S_{j+2} is issued as soon as
//              the softmax has read S_j, ahead of PV_j.
//   warp 14    TMA producer for the V ring.
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
constexpr int kAttnThreads = 512;
constexpr int kRopeWarp0 = 8;
constexpr int kTmaWarp = 12;   // Q, K (+ cos/sin rows)
constexpr int kMmaWarp = 13;
constexpr int kTmaVWarp = 14;  // V: its own producer, so K prefetch never waits on a V slot
// warp 15 only takes part in the block-wide barriers
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only if the max grows by > 2^8

struct AttnArgs {
    void* out;
    const RopeSeed* seeds;  // [sequences] in the caller's order
    int32_t layout;  // 0 BNSD, 1 TND
    int32_t B, Hq, Hkv, G;
    int32_t S;       // BNSD sequence length
    int32_t causal;
    float scale_log2;  // softmax scale * log2(e)
    int32_t n_items;
    // TND: sequences sorted by length, descending; seg_item0[k] = first work item of sequence k
    int32_t nseg;
    int32_t seg_start[16];
    int32_t seg_len[16];
    int32_t seg_tiles[16];
    int32_t seg_item0[17];
    int32_t seg_orig[16];  // caller's index of sorted sequence k
};

template <int D>
struct AttnCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kAtoms = D / 64;                 // 128-byte swizzle atoms across a row
    static constexpr int kAtomBytes = kBlockM * 128;      // one atom column of a 128-row tile
    static constexpr int kTileBytes = kBlockM * D * 2;    // Q, K or V tile
    static constexpr int kTabBytes = kBlockM * D * 2;     // cos/sin rows of a tile: D/2 fp16 cos + D/2 fp16 sin
    static constexpr int kTabBoxes = D / 64;              // 128-byte boxes of 32 (cos, sin) pairs
    static constexpr int kStages = (D == 64) ? 4 : 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kOffT = kOffV + kStages * kTileBytes;
    static constexpr int kOffBar = kOffT + kStages * kTabBytes;
    // barrier indices
    static constexpr int kBarQFull = 0, kBarQReady = 1;
    static constexpr int kBarKFull = 2;
    static constexpr int kBarVFull = kBarKFull + kStages;
    static constexpr int kBarKReady = kBarVFull + kStages;
    static constexpr int kBarKEmpty = kBarKReady + kStages;
    static constexpr int kBarVEmpty = kBarKEmpty + kStages;
    static constexpr int kBarSFull = kBarVEmpty + kStages;  // 2: S_j in TMEM buffer j % 2
    static constexpr int kBarSEmpty = kBarSFull + 2;        // 2: both warpgroups have read S_j (8 warp arrivals)
    static constexpr int kBarPFull = kBarSEmpty + 2;        // P_j written (8 warp arrivals)
    static constexpr int kBarPVDone = kBarPFull + 1;        // PV_j done: O updated, P free
    static constexpr int kBarMmaFin = kBarPVDone + 1;
    static constexpr int kBarQRot = kBarMmaFin + 1;         // Q' rotated in shared memory (4 warp arrivals)
    static constexpr int kNumBars = kBarQRot + 1;
    static constexpr int kOffAbort = kOffBar + 8 * kNumBars;
    static constexpr int kOffTmemSlot = kOffAbort + 16;
    static constexpr int kOffXchg = kOffTmemSlot + 16;  // float [2 slots][2 halves][128 rows]
    // The dynamic shared-memory window starts 1024-byte aligned on sm_100 (the
    // kernel checks it), so no alignment slack is requested.
    static constexpr int kSmemBytes = kOffXchg + 2 * 2 * kBlockM * 4;
    // TMEM columns: S/score buffers, O accumulator, Q' and P (16-bit, two per column)
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0;      // 2 x 128
    static constexpr uint32_t kColO = 256;    // D
    static constexpr uint32_t kColQ = 384;    // D / 2
    static constexpr uint32_t kColP = 448;    // 64
    static_assert(kColO + D <= kColQ && kColQ + D / 2 <= kColP && kColP + kBlockN / 2 <= kTmemCols, "TMEM budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct WorkItem {
    int32_t orig;  // sequence index in the caller's order
    int32_t tok0;  // first token of the sequence (BNSD: seq * S)
    int32_t seq;   // BNSD batch index
    int32_t L;     // sequence length
    int32_t h;     // query head
    int32_t qt;    // query tile index within the sequence
};

// Head-major order (all query tiles of one head are neighbours, so the CTAs
// resident at one time share K/V tiles through L2), largest tile first within
// a head; packed sequences longest first.
__device__ __forceinline__ WorkItem decode_item(const AttnArgs& a, int32_t x) {
    WorkItem w;
    if (a.layout == 0) {
        const int32_t nqt = (a.S + kBlockM - 1) / kBlockM;
        const int32_t bh = x / nqt;
        w.qt = nqt - 1 - (x - bh * nqt);
        w.seq = bh / a.Hq;
        w.h = bh - w.seq * a.Hq;
        w.tok0 = w.seq * a.S;
        w.L = a.S;
        w.orig = w.seq;
        return w;
    }
    int32_t s = 0;
    while (s + 1 < a.nseg && x >= a.seg_item0[s + 1]) ++s;
    const int32_t r = x - a.seg_item0[s];
    const int32_t nt = a.seg_tiles[s];
    w.h = r / nt;
    w.qt = nt - 1 - (r - w.h * nt);
    w.seq = s;
    w.orig = a.seg_orig[s];
    w.tok0 = a.seg_start[s];
    w.L = a.seg_len[s];
    return w;
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

// Rotate the first `rows` rows of a 128-row tile in shared memory with the
// cos/sin rows staged at `tab`.  128B swizzle: 16-byte chunk c of row r sits at
// r*128 + ((c ^ (r&7)) << 4) within its 128-row atom.  The table's atoms hold
// 32 (cos, sin) pairs per row, 4 pairs per chunk.
template <int D, bool kFP16>
__device__ __forceinline__ void rope_tile(uint32_t tile, uint32_t tab, int32_t rows, int32_t rt) {
    constexpr int kPairsPerRow = D / 16;  // 16-byte chunk pairs per row
    constexpr int kIters = kBlockM * kPairsPerRow / 128;
#pragma unroll 1
    for (int it = 0; it < kIters; ++it) {
        const int task = rt + 128 * it;
        const int r = task / kPairsPerRow;
        const int cp = task % kPairsPerRow;
        if (r >= rows) continue;
        const uint32_t sw = static_cast<uint32_t>(r & 7);
        uint32_t o1, o2;
        if constexpr (D == 128) {
            o1 = tile + r * 128 + ((cp ^ sw) << 4);
            o2 = o1 + AttnCfg<D>::kAtomBytes;
        } else {
            o1 = tile + r * 128 + ((cp ^ sw) << 4);
            o2 = tile + r * 128 + (((cp + 4) ^ sw) << 4);
        }
        uint4 t0, t1;
        if constexpr (D == 128) {
            // row layout of the table: chunk cp of atom 0 = pairs 8cp..8cp+3,
            // chunk cp of atom 1 = pairs 8cp+4..8cp+7 (conflict-free for the 8
            // lanes of a quarter-warp, which share a row)
            const uint32_t tb = tab + r * 128 + ((cp ^ sw) << 4);
            t0 = lds128(tb);
            t1 = lds128(tb + AttnCfg<D>::kAtomBytes);
        } else {
            const uint32_t tb = tab + r * 128;
            const uint32_t tc = static_cast<uint32_t>(cp * 2);
            t0 = lds128(tb + ((tc ^ sw) << 4));
            t1 = lds128(tb + (((tc + 1) ^ sw) << 4));
        }
        uint4 x1 = lds128(o1), x2 = lds128(o2);
        rotate8<kFP16>(x1, x2, t0, t1);
        sts128(o1, x1);
        sts128(o2, x2);
    }
}

// Angles of one RoPE thread for a key tile whose rows hold consecutive
// positions: 4 groups of 2 frequencies, (cos, sin) kept as packed fp32 pairs.
struct RecState {
    uint64_t c[4], s[4];     // current row's (cos f0, cos f1), (sin f0, sin f1)
};
// (c, s) <- (c, s) * (wc, ws) as complex numbers, two frequencies at a time
__device__ __forceinline__ void rec_step(uint64_t& c, uint64_t& s, uint64_t wc, uint64_t ws) {
    const uint64_t cn = fsub2(fmul2(c, wc), fmul2(s, ws));
    s = ffma2(s, wc, fmul2(c, ws));
    c = cn;
}

// Rotate a key tile whose rows hold consecutive positions, without a table.
// This thread's rows are r0, r0 + step, ...; z holds the angles of row r0 and
// (wc, ws) advance them by `step` rows.
template <int D, bool kFP16>
__device__ __forceinline__ void rope_tile_rec(uint32_t tile, int32_t rows, int32_t rt, const RecState& z,
                                              const uint64_t (&wc)[4], const uint64_t (&ws)[4]) {
    constexpr int kPairsPerRow = D / 16;
    constexpr int kIters = kBlockM * kPairsPerRow / 128;
    constexpr int kStep = 128 / kPairsPerRow;
    const int cp = rt % kPairsPerRow;
    const int r0 = rt / kPairsPerRow;
    RecState e = z;
    // Modest unrolling: 16 warps run four roles at once and their hot loops
    // must stay resident in the instruction cache.
#pragma unroll 2
    for (int it = 0; it < kIters; ++it) {
        const int r = r0 + it * kStep;
        if (r < rows) {
            const uint32_t sw = static_cast<uint32_t>(r & 7);
            uint32_t o1, o2;
            if constexpr (D == 128) {
                o1 = tile + r * 128 + ((cp ^ sw) << 4);
                o2 = o1 + AttnCfg<D>::kAtomBytes;
            } else {
                o1 = tile + r * 128 + ((cp ^ sw) << 4);
                o2 = tile + r * 128 + (((cp + 4) ^ sw) << 4);
            }
            uint4 x1 = lds128(o1), x2 = lds128(o2);
            uint32_t* xa = reinterpret_cast<uint32_t*>(&x1);
            uint32_t* xb = reinterpret_cast<uint32_t*>(&x2);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t X1 = IoT<kFP16>::unpack2(xa[k]);
                const uint64_t X2 = IoT<kFP16>::unpack2(xb[k]);
                xa[k] = pack2<kFP16>(fsub2(fmul2(X1, e.c[k]), fmul2(X2, e.s[k])));  // x1 cos - x2 sin
                xb[k] = pack2<kFP16>(ffma2(X2, e.c[k], fmul2(X1, e.s[k])));        // x2 cos + x1 sin
            }
            sts128(o1, x1);
            sts128(o2, x2);
        }
        if (it + 1 < kIters) {
#pragma unroll
            for (int k = 0; k < 4; ++k) rec_step(e.c[k], e.s[k], wc[k], ws[k]);
        }
    }
}

// Copy this thread's row (rt) of a rotated 128-row tile from 128B-swizzled
// shared memory into TMEM columns col0.. as packed 16-bit pairs (the A-operand
// layout of tcgen05.mma: lane = row, column c = elements 2c, 2c+1).
template <int D>
__device__ __forceinline__ void tile_row_to_tmem(uint32_t tile, uint32_t taddr, int32_t r) {
    const uint32_t sw = static_cast<uint32_t>(r & 7);
#pragma unroll 1
    for (int h = 0; h < D / 32; ++h) {  // 16 columns = 32 elements = 4 chunks per store
        uint32_t v[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int c = h * 4 + q;  // logical 16-byte chunk of the row
            const uint4 x = lds128(tile + (c >> 3) * AttnCfg<D>::kAtomBytes + r * 128 + (((c & 7) ^ sw) << 4));
            v[4 * q + 0] = x.x;
            v[4 * q + 1] = x.y;
            v[4 * q + 2] = x.z;
            v[4 * q + 3] = x.w;
        }
        tmem_st16(taddr + h * 16, v);
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

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16, A = P in TMEM.
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <int D, bool kFP16>
__global__ void __launch_bounds__(kAttnThreads, 1)
    fused_rope_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmT,
                               const __grid_constant__ AttnArgs a) {
    using C = AttnCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    if ((sbase & 1023u) != 0u) {  // 128B-swizzled TMA/UMMA tiles need 1024-byte alignment
        if (threadIdx.x == 0) record_status(2 /* RFA_ERR_UNSUPPORTED */);
        return;
    }
    uint8_t* smem = smem_raw;
    volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + C::kOffAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffTmemSlot);
    auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8u * static_cast<uint32_t>(i); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const WorkItem w = decode_item(a, blockIdx.x);
    const int32_t kvh = w.h / a.G;
    const int32_t n_kv = a.causal ? (w.qt + 1) : (w.L + kBlockN - 1) / kBlockN;
    // consecutive positions: K angles come from the recurrence, no cos/sin rows per K tile
    const bool rec = a.seeds[w.orig].consecutive != 0;

    if (threadIdx.x == 0) {
        mbar_init(bar(C::kBarQFull), 1);
        mbar_init(bar(C::kBarQReady), 4);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(bar(C::kBarKFull + s), 1);
            mbar_init(bar(C::kBarVFull + s), 1);
            mbar_init(bar(C::kBarKReady + s), 4);
            mbar_init(bar(C::kBarKEmpty + s), 1);
            mbar_init(bar(C::kBarVEmpty + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(C::kBarSFull + b), 1);
            mbar_init(bar(C::kBarSEmpty + b), 8);  // one arrival per softmax warp
        }
        mbar_init(bar(C::kBarPFull), 8);
        mbar_init(bar(C::kBarPVDone), 1);
        mbar_init(bar(C::kBarMmaFin), 1);
        mbar_init(bar(C::kBarQRot), 4);
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

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ Q/K producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmT);
            const bool bnsd = (a.layout == 0);
            const int32_t qplane = bnsd ? (w.seq * a.Hq + w.h) : w.h;
            const int32_t kvplane = bnsd ? (w.seq * a.Hkv + kvh) : kvh;
            auto load_tile = [&](const CUtensorMap* m, uint32_t dst, uint32_t b, int32_t plane, int32_t row0) {
                for (int at = 0; at < C::kAtoms; ++at) {
                    if (bnsd)
                        tma_load_3d(dst + at * C::kAtomBytes, m, b, at * 64, row0, plane);
                    else
                        tma_load_3d(dst + at * C::kAtomBytes, m, b, at * 64, plane, w.tok0 + row0);
                }
            };
            auto load_tab = [&](uint32_t dst, uint32_t b, int32_t row0) {
                for (int bx = 0; bx < C::kTabBoxes; ++bx)
                    tma_load_3d(dst + bx * C::kAtomBytes, &tmT, b, bx * 32, w.tok0 + row0, 0);
            };
            const uint32_t kbytes = C::kTileBytes + (rec ? 0 : C::kTabBytes);
            // Q and its cos/sin rows; the rows go to table stage 1, free until K tile 1.
            mbar_expect_tx(bar(C::kBarQFull), C::kTileBytes + C::kTabBytes);
            load_tile(&tmQ, sbase + C::kOffQ, bar(C::kBarQFull), qplane, w.qt * kBlockM);
            load_tab(sbase + C::kOffT + 1 * C::kTabBytes, bar(C::kBarQFull), w.qt * kBlockM);
            int32_t issued_k = 0;
            for (int32_t j = 0; j < n_kv; ++j) {
                const int s = j % C::kStages;
                const uint32_t u = static_cast<uint32_t>(j / C::kStages);
                if (!rec && j == 1 && !mbar_wait(bar(C::kBarQReady), 0, abort_flag)) break;  // Q's rows consumed
                if (u > 0 && !mbar_wait(bar(C::kBarKEmpty + s), (u - 1) & 1u, abort_flag)) break;
                mbar_expect_tx(bar(C::kBarKFull + s), kbytes);
                load_tile(&tmK, sbase + C::kOffK + s * C::kTileBytes, bar(C::kBarKFull + s), kvplane, j * kBlockN);
                if (!rec) load_tab(sbase + C::kOffT + s * C::kTabBytes, bar(C::kBarKFull + s), j * kBlockN);
                issued_k = j + 1;
            }
            // Drain: every issued copy must have landed before the CTA exits.
            mbar_wait_drain(bar(C::kBarQFull), 0);
            for (int32_t j = (issued_k > C::kStages ? issued_k - C::kStages : 0); j < issued_k; ++j)
                mbar_wait_drain(bar(C::kBarKFull + j % C::kStages), static_cast<uint32_t>(j / C::kStages) & 1u);
        }
    } else if (warp == kTmaVWarp) {
        // ------------------------------------------------------------ V producer
        if (lane == 0) {
            tma_prefetch_desc(&tmV);
            const bool bnsd = (a.layout == 0);
            const int32_t kvplane = bnsd ? (w.seq * a.Hkv + kvh) : kvh;
            int32_t issued_v = 0;
            for (int32_t j = 0; j < n_kv; ++j) {
                const int s = j % C::kStages;
                const uint32_t u = static_cast<uint32_t>(j / C::kStages);
                if (u > 0 && !mbar_wait(bar(C::kBarVEmpty + s), (u - 1) & 1u, abort_flag)) break;
                mbar_expect_tx(bar(C::kBarVFull + s), C::kTileBytes);
                const uint32_t dst = sbase + C::kOffV + s * C::kTileBytes;
                for (int at = 0; at < C::kAtoms; ++at) {
                    if (bnsd)
                        tma_load_3d(dst + at * C::kAtomBytes, &tmV, bar(C::kBarVFull + s), at * 64, j * kBlockN, kvplane);
                    else
                        tma_load_3d(dst + at * C::kAtomBytes, &tmV, bar(C::kBarVFull + s), at * 64, kvplane,
                                    w.tok0 + j * kBlockN);
                }
                issued_v = j + 1;
            }
            for (int32_t j = (issued_v > C::kStages ? issued_v - C::kStages : 0); j < issued_v; ++j)
                mbar_wait_drain(bar(C::kBarVFull + j % C::kStages), static_cast<uint32_t>(j / C::kStages) & 1u);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ tcgen05 issuer
        if (lane == 0) {
            constexpr uint32_t kIdescQK = idesc_f16(IoT<kFP16>::kFmt, 0, 0, kBlockM, kBlockN);
            constexpr uint32_t kIdescPV = idesc_f16(IoT<kFP16>::kFmt, 0, 1, kBlockM, D);
            auto issue_qk = [&](int32_t j) -> bool {
                const int s = j % C::kStages;
                const int b = j & 1;
                if (!mbar_wait(bar(C::kBarKReady + s), static_cast<uint32_t>(j / C::kStages) & 1u, abort_flag))
                    return false;
                // buffer b held S_{j-2}: both softmax warpgroups must have read it
                if (j >= 2 && !mbar_wait(bar(C::kBarSEmpty + b), static_cast<uint32_t>((j >> 1) - 1) & 1u, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t kbase = sbase + C::kOffK + s * C::kTileBytes;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t koff = (k >> 2) * C::kAtomBytes + (k & 3) * 32;
                    const uint64_t bd = smem_desc_sw128(kbase + koff, 16, 1024);
                    // A = Q' from TMEM: 16 elements of K = 8 packed columns per step
                    umma_ts(tmem + C::kColS + b * kBlockN, tmem + C::kColQ + k * 8, bd, kIdescQK, k > 0 ? 1u : 0u);
                }
                tc_commit(bar(C::kBarSFull + b));
                tc_commit(bar(C::kBarKEmpty + s));
                return true;
            };
            auto issue_pv = [&](int32_t i) -> bool {
                const int s = i % C::kStages;
                if (!mbar_wait(bar(C::kBarPFull), static_cast<uint32_t>(i) & 1u, abort_flag)) return false;
                if (!mbar_wait(bar(C::kBarVFull + s), static_cast<uint32_t>(i / C::kStages) & 1u, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t vbase = sbase + C::kOffV + s * C::kTileBytes;
#pragma unroll
                for (int k = 0; k < kBlockN / 16; ++k) {
                    const uint64_t bd = smem_desc_sw128(vbase + k * 16 * 128, C::kAtomBytes, 1024);
                    umma_ts(tmem + C::kColO, tmem + C::kColP + k * 8, bd, kIdescPV, (i > 0 || k > 0) ? 1u : 0u);
                }
                tc_commit(bar(C::kBarPVDone));
                tc_commit(bar(C::kBarVEmpty + s));
                return true;
            };
            bool ok = mbar_wait(bar(C::kBarQReady), 0, abort_flag);
            if (ok) {
                tc_fence_after();
                ok = issue_qk(0);
                if (ok && n_kv > 1) ok = issue_qk(1);
                for (int32_t j = 0; j < n_kv && ok; ++j) {
                    if (j + 2 < n_kv) ok = issue_qk(j + 2);
                    if (ok) ok = issue_pv(j);
                }
            }
            tc_commit(bar(C::kBarMmaFin));
            mbar_wait_drain(bar(C::kBarMmaFin), 0);
        }
    } else if (warp >= kRopeWarp0 && warp < kRopeWarp0 + 4) {
        // ------------------------------------------------------------ RoPE warpgroup
        const int32_t rt = threadIdx.x - kRopeWarp0 * 32;  // == TMEM lane of this thread
        constexpr int kPairsPerRow = D / 16;
        RecState z;
        uint64_t wc[4], ws[4], wc128[4], ws128[4];
        if (rec) {
            const RopeSeed* sd = a.seeds + w.orig;
            const int cp = rt % kPairsPerRow;
            const int r0 = rt / kPairsPerRow;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int f = 8 * cp + 2 * k;
                float2 z0 = sd->z0[r0 % kSeedRows][f], z1 = sd->z0[r0 % kSeedRows][f + 1];
                const float2 w0 = sd->w16[f], w1 = sd->w16[f + 1];
                wc[k] = f2pack(w0.x, w1.x);
                ws[k] = f2pack(w0.y, w1.y);
                z.c[k] = f2pack(z0.x, z1.x);
                z.s[k] = f2pack(z0.y, z1.y);
                if (r0 >= kSeedRows) rec_step(z.c[k], z.s[k], wc[k], ws[k]);  // D = 64: rows 16..31
                if (D == 64) {  // D = 64 steps by 32 rows: w32 = w16^2
                    uint64_t c2 = wc[k], s2 = ws[k];
                    rec_step(c2, s2, wc[k], ws[k]);
                    wc[k] = c2;
                    ws[k] = s2;
                }
                const float2 v0 = sd->w128[f], v1 = sd->w128[f + 1];
                wc128[k] = f2pack(v0.x, v1.x);
                ws128[k] = f2pack(v0.y, v1.y);
            }
        }
        if (mbar_wait(bar(C::kBarQFull), 0, abort_flag)) {
            const int32_t q0 = w.qt * kBlockM;
            rope_tile<D, kFP16>(sbase + C::kOffQ, sbase + C::kOffT + 1 * C::kTabBytes, min(kBlockM, w.L - q0), rt);
            // all of Q' rotated (by every RoPE warp) before rows are copied to TMEM
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarQRot));
            const bool qrot = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarQRot), 0, abort_flag));
            if (qrot) {
                tile_row_to_tmem<D>(sbase + C::kOffQ, tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + C::kColQ, rt);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::kBarQReady));
            }
            for (int32_t j = 0; j < n_kv && qrot; ++j) {
                const int s = j % C::kStages;
                const uint32_t u = static_cast<uint32_t>(j / C::kStages);
                if (!mbar_wait(bar(C::kBarKFull + s), u & 1u, abort_flag)) break;
                const int32_t k0 = j * kBlockN;
                if (rec) {
                    rope_tile_rec<D, kFP16>(sbase + C::kOffK + s * C::kTileBytes, min(kBlockN, w.L - k0), rt, z, wc, ws);
#pragma unroll
                    for (int k = 0; k < 4; ++k) rec_step(z.c[k], z.s[k], wc128[k], ws128[k]);
                } else {
                    rope_tile<D, kFP16>(sbase + C::kOffK + s * C::kTileBytes, sbase + C::kOffT + s * C::kTabBytes,
                                        min(kBlockN, w.L - k0), rt);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::kBarKReady + s));
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax warpgroups
        // The two warpgroups meet at named barrier 1 exactly n_kv + 1 times: a
        // failed (timed-out) wait only turns the remaining work into no-ops,
        // it never skips a barrier, so the barrier cannot deadlock.
        const int hf = warp >> 2;            // key-column half of every score tile
        const int row = threadIdx.x & 127;   // 0..127 == TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        float* xmax = reinterpret_cast<float*>(smem + C::kOffXchg);  // [slot][half][row]
        const int32_t qi = w.qt * kBlockM + row;
        const float sl2 = a.scale_log2;
        constexpr int kOHalf = D / 2;        // O columns rescaled / stored by this warpgroup
        float m = -INFINITY;  // running max of score * scale * log2(e) (same in both warpgroups)
        float l = 0.0f;       // this half's running sum of exp2(score * scale_log2 - m)
        bool ok = true;       // warp-uniform
        for (int32_t j = 0; j < n_kv; ++j) {
            const int b = j & 1;
            const int slot = j & 1;
            // tcgen05.ld/st are warp-collective: every decision below is warp-uniform.
            ok = ok && __all_sync(0xffffffffu, mbar_wait(bar(C::kBarSFull + b), static_cast<uint32_t>(j >> 1) & 1u,
                                                         abort_flag));
            uint32_t sr[2][32];
            float mxh = -INFINITY;
            if (ok) {
                tc_fence_after();
                const uint32_t sc = tmem + lane_off + C::kColS + b * kBlockN + hf * 64;
                tmem_ld32(sc, sr[0]);
                tmem_ld32(sc + 32, sr[1]);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::kBarSEmpty + b));  // S_j consumed: the buffer may take S_{j+2}

                // mask: keys [kv0, kv0 + lim) of this half are visible to this row
                const int32_t kv0 = j * kBlockN + hf * 64;
                const int32_t lim = (a.causal ? min(qi + 1, w.L) : w.L) - kv0;
                if (lim < 64) {
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (c >= lim) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
                }
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c = 0; c < 64; c += 2)
                    mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(sr[c >> 5][c & 31]),
                                              __uint_as_float(sr[c >> 5][(c + 1) & 31]));
                mxh = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
            }
            // exchange half-row maxima with the other warpgroup
            xmax[(slot * 2 + hf) * kBlockM + row] = mxh;
            named_bar_sync(1, 256);
            ok = __all_sync(0xffffffffu, ok && *abort_flag == 0);
            if (!ok) continue;
            const float mx = fmaxf(mxh, xmax[(slot * 2 + (hf ^ 1)) * kBlockM + row]);
            const float m_new = fmaxf(m, mx * sl2);
            // PV_{j-1} must be done before P_j overwrites P_{j-1} (and before O is rescaled)
            if (j > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarPVDone), static_cast<uint32_t>(j - 1) & 1u, abort_flag));
                if (!ok) continue;
                tc_fence_after();
                const bool need = m_new > m + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need)) {
                    const float alpha = need ? ex2(m - m_new) : 1.0f;
                    const uint64_t alpha2 = f2pack(alpha, alpha);
                    l *= alpha;
#pragma unroll 1
                    for (int q = 0; q < kOHalf / 32; ++q) {
                        uint32_t o[32];
                        const uint32_t oc = tmem + lane_off + C::kColO + hf * kOHalf + q * 32;
                        tmem_ld32(oc, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; c += 2) {
                            const float2 v = f2unpack(fmul2(f2pack(__uint_as_float(o[c]), __uint_as_float(o[c + 1])), alpha2));
                            o[c] = __float_as_uint(v.x);
                            o[c + 1] = __float_as_uint(v.y);
                        }
                        tmem_st32(oc, o);
                    }
                    if (need) m = m_new;
                }
            } else {
                m = m_new;
            }
            const float neg_m = (m == -INFINITY) ? 0.0f : -m;
            uint32_t pw[32];
            const uint64_t sl2x2 = f2pack(sl2, sl2), negm2 = f2pack(neg_m, neg_m);
            uint64_t l2[2] = {0ull, 0ull};  // packed (+0.0f, +0.0f)
#pragma unroll
            for (int c2 = 0; c2 < 32; ++c2) {
                const int c = 2 * c2;
                const uint64_t sv = f2pack(__uint_as_float(sr[c >> 5][c & 31]), __uint_as_float(sr[c >> 5][(c + 1) & 31]));
                const float2 x = f2unpack(ffma2(sv, sl2x2, negm2));
                const uint64_t pp = f2pack(ex2(x.x), ex2(x.y));
                l2[c2 & 1] = fadd2(l2[c2 & 1], pp);
                pw[c2] = pack2<kFP16>(pp);
            }
            const float2 la = f2unpack(fadd2(l2[0], l2[1]));
            l += la.x + la.y;
            tmem_st32(tmem + lane_off + C::kColP + hf * 32, pw);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarPFull));
        }
        // epilogue: combine the partial sums (one more named barrier), out = O / l after the last PV
        {
            const int slot = n_kv & 1;  // last read at tile n_kv-2, free for both warpgroups now
            xmax[(slot * 2 + hf) * kBlockM + row] = l;
            named_bar_sync(1, 256);
            l += xmax[(slot * 2 + (hf ^ 1)) * kBlockM + row];
        }
        const bool fin = __all_sync(0xffffffffu, ok && *abort_flag == 0) &&
                         __all_sync(0xffffffffu, mbar_wait(bar(C::kBarPVDone), static_cast<uint32_t>(n_kv - 1) & 1u,
                                                           abort_flag));
        if (fin) {
            tc_fence_after();
            const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
            const bool valid = qi < w.L;
            uint16_t* outp = reinterpret_cast<uint16_t*>(a.out);
            int64_t o_off;
            if (a.layout == 0)
                o_off = ((static_cast<int64_t>(w.seq) * a.Hq + w.h) * a.S + qi) * D;
            else
                o_off = (static_cast<int64_t>(w.tok0 + qi) * a.Hq + w.h) * D;
            o_off += hf * kOHalf;
            const uint64_t il2 = f2pack(inv_l, inv_l);
#pragma unroll 1
            for (int q = 0; q < kOHalf / 32; ++q) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + C::kColO + hf * kOHalf + q * 32, o);
                tmem_wait_ld();
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(outp + o_off + q * 32);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint32_t wv[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c = 8 * v4 + 2 * e;
                            wv[e] = pack2<kFP16>(fmul2(f2pack(__uint_as_float(o[c]), __uint_as_float(o[c + 1])), il2));
                        }
                        dst[v4] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                    }
                }
            }
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace rfa
