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
//              mask, exchange the half-row maxima through shared memory, keep
//              the running max (identical in both) and a partial sum, write P
//              (bf16/fp16) back into TMEM, rescale its half of O only when the
//              max grows by > 2^8.  At the end the partial sums are combined
//              and each warpgroup normalises and stores half of the columns.
//   warps 8-11 RoPE warpgroup: rotates the Q tile once and every K tile in
//              place in the 128B-swizzled shared-memory layout, reading the
//              cos/sin rows that TMA staged next to the tile.  Element i and
//              its rotate-half partner i + D/2 sit at the same offset of two
//              swizzle atoms (D = 128) or in chunks c and c ^ 4 of one atom
//              (D = 64), so each thread rotates 8 pairs per 2 x 16 B.
//   warp 12    TMA producer: Q (+ its cos/sin rows) once, then K (+ cos/sin)
//              tiles through a kStages ring.
//   warp 14    TMA producer for the V ring (V slots free up later than K
//              slots, so one producer for both would hold back K prefetch).
//   warp 13    tcgen05 issuer (one thread) and TMEM owner.  S_j = Q'K_j'^T goes
//              to TMEM buffer j % 3; O += P_j V_j reads P_j from that buffer
//              (A operand in TMEM) and V_j from shared memory.  QK runs two
//              tiles ahead of PV so the softmax never waits for its scores.
// Completion of every async step is tracked by mbarriers; each wait is bounded.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

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
constexpr int kSBufs = 3;                  // S/P buffers in TMEM
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only if the max grows by > 2^8

struct AttnArgs {
    void* out;
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
};

template <int D>
struct AttnCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kAtoms = D / 64;                 // 128-byte swizzle atoms across a row
    static constexpr int kAtomBytes = kBlockM * 128;      // one atom column of a 128-row tile
    static constexpr int kTileBytes = kBlockM * D * 2;    // Q, K or V tile
    static constexpr int kTabBytes = kBlockM * D * 2;     // cos/sin rows of a tile: D/2 fp16 pairs per row
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
    static constexpr int kBarSFull = kBarVEmpty + kStages;  // kSBufs
    static constexpr int kBarPFull = kBarSFull + kSBufs;    // kSBufs
    static constexpr int kBarBufFree = kBarPFull + kSBufs;  // kSBufs: PV of that buffer done
    static constexpr int kBarMmaFin = kBarBufFree + kSBufs;
    static constexpr int kBarXchg = kBarMmaFin + 1;  // 2: half-row maxima exchanged (256 arrivals)
    static constexpr int kNumBars = kBarXchg + 2;
    static constexpr int kOffAbort = kOffBar + 8 * kNumBars;
    static constexpr int kOffTmemSlot = kOffAbort + 16;
    static constexpr int kOffXchg = kOffTmemSlot + 16;  // float [2 slots][2 halves][128 rows]
    // The dynamic shared-memory window starts 1024-byte aligned on sm_100 (the
    // kernel checks it), so no alignment slack is requested.
    static constexpr int kSmemBytes = kOffXchg + 2 * 2 * kBlockM * 4;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColO = kSBufs * kBlockN;  // S/P buffers at 0, 128, 256; O at 384
    static_assert(kColO + D <= kTmemCols, "TMEM budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct WorkItem {
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
        return w;
    }
    int32_t s = 0;
    while (s + 1 < a.nseg && x >= a.seg_item0[s + 1]) ++s;
    const int32_t r = x - a.seg_item0[s];
    const int32_t nt = a.seg_tiles[s];
    w.h = r / nt;
    w.qt = nt - 1 - (r - w.h * nt);
    w.seq = s;
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
#pragma unroll 4
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
        for (int b = 0; b < kSBufs; ++b) {
            mbar_init(bar(C::kBarSFull + b), 1);
            mbar_init(bar(C::kBarPFull + b), 8);
            mbar_init(bar(C::kBarBufFree + b), 1);
        }
        mbar_init(bar(C::kBarMmaFin), 1);
        mbar_init(bar(C::kBarXchg + 0), 256);
        mbar_init(bar(C::kBarXchg + 1), 256);
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
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
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
            // Q and its cos/sin rows; the rows go to table stage 1, free until K tile 1.
            mbar_expect_tx(bar(C::kBarQFull), C::kTileBytes + C::kTabBytes);
            load_tile(&tmQ, sbase + C::kOffQ, bar(C::kBarQFull), qplane, w.qt * kBlockM);
            load_tab(sbase + C::kOffT + 1 * C::kTabBytes, bar(C::kBarQFull), w.qt * kBlockM);
            int32_t issued_k = 0;
            for (int32_t j = 0; j < n_kv; ++j) {
                const int s = j % C::kStages;
                const uint32_t u = static_cast<uint32_t>(j / C::kStages);
                if (j == 1 && !mbar_wait(bar(C::kBarQReady), 0, abort_flag)) break;  // Q's rows consumed
                if (u > 0 && !mbar_wait(bar(C::kBarKEmpty + s), (u - 1) & 1u, abort_flag)) break;
                mbar_expect_tx(bar(C::kBarKFull + s), C::kTileBytes + C::kTabBytes);
                load_tile(&tmK, sbase + C::kOffK + s * C::kTileBytes, bar(C::kBarKFull + s), kvplane, j * kBlockN);
                load_tab(sbase + C::kOffT + s * C::kTabBytes, bar(C::kBarKFull + s), j * kBlockN);
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
                const int b = j % kSBufs;
                if (!mbar_wait(bar(C::kBarKReady + s), static_cast<uint32_t>(j / C::kStages) & 1u, abort_flag))
                    return false;
                // the buffer held P_{j-3}: PV_{j-3} must have read it
                if (j >= kSBufs && !mbar_wait(bar(C::kBarBufFree + b), static_cast<uint32_t>(j / kSBufs - 1) & 1u,
                                              abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t kbase = sbase + C::kOffK + s * C::kTileBytes;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t koff = (k >> 2) * C::kAtomBytes + (k & 3) * 32;
                    const uint64_t ad = smem_desc_sw128(sbase + C::kOffQ + koff, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(kbase + koff, 16, 1024);
                    umma_ss(tmem + b * kBlockN, ad, bd, kIdescQK, k > 0 ? 1u : 0u);
                }
                tc_commit(bar(C::kBarSFull + b));
                tc_commit(bar(C::kBarKEmpty + s));
                return true;
            };
            auto issue_pv = [&](int32_t i) -> bool {
                const int s = i % C::kStages;
                const int b = i % kSBufs;
                if (!mbar_wait(bar(C::kBarPFull + b), static_cast<uint32_t>(i / kSBufs) & 1u, abort_flag))
                    return false;
                if (!mbar_wait(bar(C::kBarVFull + s), static_cast<uint32_t>(i / C::kStages) & 1u, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t vbase = sbase + C::kOffV + s * C::kTileBytes;
#pragma unroll
                for (int k = 0; k < kBlockN / 16; ++k) {
                    // P_i: 128 x 128 fp16/bf16 packed two per 32-bit column -> 8 columns per K=16 step
                    const uint64_t bd = smem_desc_sw128(vbase + k * 16 * 128, C::kAtomBytes, 1024);
                    umma_ts(tmem + C::kColO, tmem + b * kBlockN + k * 8, bd, kIdescPV, (i > 0 || k > 0) ? 1u : 0u);
                }
                tc_commit(bar(C::kBarBufFree + b));
                tc_commit(bar(C::kBarVEmpty + s));
                return true;
            };
            bool ok = mbar_wait(bar(C::kBarQReady), 0, abort_flag);
            if (ok) {
                tc_fence_after();
                ok = issue_qk(0);
                if (ok && n_kv > 1) ok = issue_qk(1);
                for (int32_t j = 0; j < n_kv && ok; ++j) {
                    ok = issue_pv(j);
                    if (ok && j + 2 < n_kv) ok = issue_qk(j + 2);
                }
            }
            tc_commit(bar(C::kBarMmaFin));
            mbar_wait_drain(bar(C::kBarMmaFin), 0);
        }
    } else if (warp >= kRopeWarp0 && warp < kRopeWarp0 + 4) {
        // ------------------------------------------------------------ RoPE warpgroup
        const int32_t rt = threadIdx.x - kRopeWarp0 * 32;
        if (mbar_wait(bar(C::kBarQFull), 0, abort_flag)) {
            const int32_t q0 = w.qt * kBlockM;
            rope_tile<D, kFP16>(sbase + C::kOffQ, sbase + C::kOffT + 1 * C::kTabBytes, min(kBlockM, w.L - q0), rt);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarQReady));
            for (int32_t j = 0; j < n_kv; ++j) {
                const int s = j % C::kStages;
                const uint32_t u = static_cast<uint32_t>(j / C::kStages);
                if (!mbar_wait(bar(C::kBarKFull + s), u & 1u, abort_flag)) break;
                const int32_t k0 = j * kBlockN;
                rope_tile<D, kFP16>(sbase + C::kOffK + s * C::kTileBytes, sbase + C::kOffT + s * C::kTabBytes,
                                    min(kBlockN, w.L - k0), rt);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::kBarKReady + s));
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax warpgroups
        const int hf = warp >> 2;            // key-column half of every score tile
        const int row = threadIdx.x & 127;   // 0..127 == TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        float* xmax = reinterpret_cast<float*>(smem + C::kOffXchg);  // [slot][half][row]
        const int32_t qi = w.qt * kBlockM + row;
        const float sl2 = a.scale_log2;
        constexpr int kOHalf = D / 2;        // O columns rescaled / stored by this warpgroup
        float m = -INFINITY;  // running max of score * scale * log2(e) (same in both warpgroups)
        float l = 0.0f;       // this half's running sum of exp2(score * scale_log2 - m)
        bool ok = true;
        for (int32_t j = 0; j < n_kv; ++j) {
            const int b = j % kSBufs;
            // tcgen05.ld/st are warp-collective: every decision below is warp-uniform.
            if (!__all_sync(0xffffffffu, mbar_wait(bar(C::kBarSFull + b), static_cast<uint32_t>(j / kSBufs) & 1u,
                                                   abort_flag))) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[2][32];
            const uint32_t sc = tmem + lane_off + b * kBlockN + hf * 64;
            tmem_ld32(sc, sr[0]);
            tmem_ld32(sc + 32, sr[1]);
            tmem_wait_ld();

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
            const float mxh = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
            // exchange half-row maxima with the other warpgroup
            const int slot = j & 1;
            xmax[(slot * 2 + hf) * kBlockM + row] = mxh;
            mbar_arrive(bar(C::kBarXchg + slot));
            if (!__all_sync(0xffffffffu, mbar_wait(bar(C::kBarXchg + slot), static_cast<uint32_t>(j >> 1) & 1u,
                                                   abort_flag))) { ok = false; break; }
            const float mx = fmaxf(mxh, xmax[(slot * 2 + (hf ^ 1)) * kBlockM + row]);
            const float m_new = fmaxf(m, mx * sl2);
            if (j > 0) {
                const bool need = m_new > m + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need)) {
                    // O holds the sum up to tile j-1 only once PV_{j-1} is done.
                    const int pb = (j - 1) % kSBufs;
                    if (!__all_sync(0xffffffffu, mbar_wait(bar(C::kBarBufFree + pb),
                                                           static_cast<uint32_t>((j - 1) / kSBufs) & 1u,
                                                           abort_flag))) { ok = false; break; }
                    tc_fence_after();
                    const float alpha = need ? ex2(m - m_new) : 1.0f;
                    l *= alpha;
#pragma unroll 1
                    for (int q = 0; q < kOHalf / 32; ++q) {
                        uint32_t o[32];
                        const uint32_t oc = tmem + lane_off + C::kColO + hf * kOHalf + q * 32;
                        tmem_ld32(oc, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                        tmem_st32(oc, o);
                    }
                    if (need) m = m_new;
                }
            } else {
                m = m_new;
            }
            const float neg_m = (m == -INFINITY) ? 0.0f : -m;
            // P_j (this half: 32 packed columns) overwrites S_j columns that both
            // warpgroups have already loaded (the exchange above orders it).
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
            tmem_st32(tmem + lane_off + b * kBlockN + hf * 32, pw);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarPFull + b));
        }
        // epilogue: combine the partial sums, out = O / l after the last PV
        bool fin = ok;
        if (fin) {
            const int slot = n_kv & 1;  // last read at tile n_kv-2, free for both warpgroups now
            xmax[(slot * 2 + hf) * kBlockM + row] = l;
            mbar_arrive(bar(C::kBarXchg + slot));
            fin = mbar_wait(bar(C::kBarXchg + slot), static_cast<uint32_t>(n_kv >> 1) & 1u, abort_flag);
            if (fin) l += xmax[(slot * 2 + (hf ^ 1)) * kBlockM + row];
        }
        const int lb = (n_kv - 1) % kSBufs;
        fin = fin && mbar_wait(bar(C::kBarBufFree + lb), static_cast<uint32_t>((n_kv - 1) / kSBufs) & 1u, abort_flag);
        if (__all_sync(0xffffffffu, fin)) {
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
#pragma unroll 1
            for (int q = 0; q < kOHalf / 32; ++q) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + C::kColO + hf * kOHalf + q * 32, o);
                tmem_wait_ld();
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(outp + o_off + q * 32);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 v;
                        v.x = IoT<kFP16>::pack(__uint_as_float(o[8 * v4 + 0]) * inv_l, __uint_as_float(o[8 * v4 + 1]) * inv_l);
                        v.y = IoT<kFP16>::pack(__uint_as_float(o[8 * v4 + 2]) * inv_l, __uint_as_float(o[8 * v4 + 3]) * inv_l);
                        v.z = IoT<kFP16>::pack(__uint_as_float(o[8 * v4 + 4]) * inv_l, __uint_as_float(o[8 * v4 + 5]) * inv_l);
                        v.w = IoT<kFP16>::pack(__uint_as_float(o[8 * v4 + 6]) * inv_l, __uint_as_float(o[8 * v4 + 7]) * inv_l);
                        dst[v4] = v;
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
