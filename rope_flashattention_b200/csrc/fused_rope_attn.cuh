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
//   warps 0-3  softmax warpgroup: thread t owns query row t of the tile (TMEM
//              lane t).  Reads S from TMEM, masks, keeps the running max and
//              sum, rescales O in TMEM only when the max grows by > 2^8,
//              writes P (bf16/fp16) to shared memory, and at the end
//              normalises O and stores the output row.
//   warps 4-7  RoPE warpgroup: rotates the Q tile once and every K tile in
//              place in the 128B-swizzled shared-memory layout.  Element i and
//              its rotate-half partner i + D/2 sit at the same offset of two
//              swizzle atoms (D = 128) or in chunks c and c ^ 4 of one atom
//              (D = 64), so each thread rotates 8 pairs per 2 x 16 B.
//   warp 8     TMA producer: Q once, K/V tiles through a kStages ring.
//   warp 9     tcgen05 issuer (one thread): S = Q'K'^T into one of two TMEM S
//              buffers, O += P V into TMEM; completion signalled by
//              tcgen05.commit onto mbarriers.  Also allocates TMEM.
// The issue order QK(j), PV(j-1) lets the tensor core compute the next score
// tile while the softmax warpgroup works on the current one.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace rfa {

constexpr int kBlockM = 128;  // query rows per tile (= TMEM lanes)
constexpr int kBlockN = 128;  // keys per tile
constexpr int kAttnThreads = 320;
constexpr int kRopeWarp0 = 4;
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only if the max grows by > 2^8

struct AttnArgs {
    void* out;
    const float* table;  // [T][2][D/2]: cos then sin, fp32
    int32_t layout;      // 0 BNSD, 1 TND
    int32_t B, Hq, Hkv, G;
    int32_t S;           // BNSD sequence length
    int32_t causal;
    float scale_log2;    // softmax scale * log2(e)
    int32_t n_items;
    // TND: sequences sorted by query-tile count, descending
    int32_t nseg;
    int32_t seg_start[16];
    int32_t seg_len[16];
    int32_t seg_tiles[16];
};

template <int D>
struct AttnCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kAtoms = D / 64;                    // 128-byte swizzle atoms across a row
    static constexpr int kAtomBytes = kBlockM * 128;         // one atom column of a 128-row tile
    static constexpr int kTileBytes = kBlockM * D * 2;       // Q, K or V tile
    static constexpr int kStages = (D == 64) ? 4 : 2;
    static constexpr int kPBytes = kBlockM * kBlockN * 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kOffP = kOffV + kStages * kTileBytes;
    static constexpr int kOffBar = kOffP + kPBytes;
    // barrier indices
    static constexpr int kBarQFull = 0, kBarQReady = 1;
    static constexpr int kBarKFull = 2;
    static constexpr int kBarVFull = kBarKFull + kStages;
    static constexpr int kBarKReady = kBarVFull + kStages;
    static constexpr int kBarKEmpty = kBarKReady + kStages;
    static constexpr int kBarVEmpty = kBarKEmpty + kStages;
    static constexpr int kBarSFull = kBarVEmpty + kStages;   // 2
    static constexpr int kBarSEmpty = kBarSFull + 2;         // 2
    static constexpr int kBarPFull = kBarSEmpty + 2;
    static constexpr int kBarPVDone = kBarPFull + 1;
    static constexpr int kBarMmaFin = kBarPVDone + 1;
    static constexpr int kNumBars = kBarMmaFin + 1;
    static constexpr int kOffAbort = kOffBar + 8 * kNumBars;
    static constexpr int kOffTmemSlot = kOffAbort + 16;
    static constexpr int kSmemBytes = kOffTmemSlot + 16 + 1024;  // + slack for 1024-byte alignment
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0;    // S buffers at columns 0 and 128
    static constexpr uint32_t kColO = 256;  // O at columns 256 .. 256+D
};

struct WorkItem {
    int32_t tok0;  // first token of the sequence (BNSD: seq * S)
    int32_t seq;   // BNSD batch index (unused for TND addressing)
    int32_t L;     // sequence length
    int32_t h;     // query head
    int32_t qt;    // query tile index within the sequence
};

// Longest-first order: all items of the highest query-tile index come first.
__device__ __forceinline__ WorkItem decode_item(const AttnArgs& a, int32_t x) {
    WorkItem w;
    if (a.layout == 0) {
        const int32_t nqt = (a.S + kBlockM - 1) / kBlockM;
        const int32_t per = a.B * a.Hq;
        const int32_t t = x / per;
        const int32_t r = x - t * per;
        w.qt = nqt - 1 - t;
        w.seq = r / a.Hq;
        w.h = r - w.seq * a.Hq;
        w.tok0 = w.seq * a.S;
        w.L = a.S;
        return w;
    }
    int32_t rem = x;
    for (int32_t k = 0; k < a.nseg; ++k) {
        const int32_t nk = a.seg_tiles[k];
        const int32_t nk1 = (k + 1 < a.nseg) ? a.seg_tiles[k + 1] : 0;
        const int32_t width = (k + 1) * a.Hq;  // items per query-tile index in this band
        const int32_t cnt = (nk - nk1) * width;
        if (rem < cnt) {
            const int32_t tt = rem / width;
            const int32_t r = rem - tt * width;
            const int32_t s = r / a.Hq;
            w.qt = nk - 1 - tt;
            w.h = r - s * a.Hq;
            w.seq = s;
            w.tok0 = a.seg_start[s];
            w.L = a.seg_len[s];
            return w;
        }
        rem -= cnt;
    }
    w.qt = -1;  // unreachable for x < n_items
    w.seq = w.h = w.tok0 = w.L = 0;
    return w;
}

template <bool kFP16>
struct IoT;
template <>
struct IoT<false> {
    static __device__ __forceinline__ float2 unpack(uint32_t u) {
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
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
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static constexpr uint32_t kFmt = 0;
};

// Rotate 8 rotate-half pairs held in two 16-byte chunks (x1: dims i..i+7,
// x2: dims i+D/2..i+D/2+7), angles from cos[0..7], sin[0..7].
template <bool kFP16>
__device__ __forceinline__ void rotate8(uint4& x1, uint4& x2, const float* cs, const float* sn) {
    uint32_t* a = reinterpret_cast<uint32_t*>(&x1);
    uint32_t* b = reinterpret_cast<uint32_t*>(&x2);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 u = IoT<kFP16>::unpack(a[k]);
        const float2 v = IoT<kFP16>::unpack(b[k]);
        const float c0 = cs[2 * k], c1 = cs[2 * k + 1], s0 = sn[2 * k], s1 = sn[2 * k + 1];
        const float y10 = u.x * c0 - v.x * s0, y11 = u.y * c1 - v.y * s1;
        const float y20 = v.x * c0 + u.x * s0, y21 = v.y * c1 + u.y * s1;
        a[k] = IoT<kFP16>::pack(y10, y11);
        b[k] = IoT<kFP16>::pack(y20, y21);
    }
}

// Rotate the first `rows` rows of a 128-row tile in shared memory (128B
// swizzle: 16-byte chunk c of row r sits at r*128 + ((c ^ (r&7)) << 4) within
// its atom).  table_row0 points at the cos/sin row of the tile's first token.
template <int D, bool kFP16>
__device__ __forceinline__ void rope_tile(uint32_t tile, int32_t rows, const float* __restrict__ table_row0,
                                          int32_t rt) {
    constexpr int kHalf = D / 2;
    constexpr int kPairsPerRow = kHalf / 8;             // 16-byte chunk pairs per row
    constexpr int kIters = kBlockM * kPairsPerRow / 128;
#pragma unroll 2
    for (int it = 0; it < kIters; ++it) {
        const int task = rt + 128 * it;
        const int r = task / kPairsPerRow;
        const int cp = task % kPairsPerRow;
        if (r >= rows) continue;
        const float* row = table_row0 + static_cast<int64_t>(r) * D;  // [cos(half) | sin(half)]
        const float4* c4 = reinterpret_cast<const float4*>(row + 8 * cp);
        const float4* s4 = reinterpret_cast<const float4*>(row + kHalf + 8 * cp);
        const float4 ca = __ldg(c4), cb = __ldg(c4 + 1), sa = __ldg(s4), sb = __ldg(s4 + 1);
        const float cs[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
        const float sn[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
        uint32_t o1, o2;
        if constexpr (D == 128) {
            o1 = tile + r * 128 + ((cp ^ (r & 7)) << 4);
            o2 = o1 + AttnCfg<D>::kAtomBytes;
        } else {
            o1 = tile + r * 128 + ((cp ^ (r & 7)) << 4);
            o2 = tile + r * 128 + (((cp + 4) ^ (r & 7)) << 4);
        }
        uint4 x1 = lds128(o1), x2 = lds128(o2);
        rotate8<kFP16>(x1, x2, cs, sn);
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

template <int D, bool kFP16>
__global__ void __launch_bounds__(kAttnThreads, 1)
    fused_rope_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnArgs a) {
    using C = AttnCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw);
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
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(C::kBarSFull + b), 1);
            mbar_init(bar(C::kBarSEmpty + b), 4);
        }
        mbar_init(bar(C::kBarPFull), 4);
        mbar_init(bar(C::kBarPVDone), 1);
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

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            const bool bnsd = (a.layout == 0);
            const int32_t qplane = bnsd ? (w.seq * a.Hq + w.h) : w.h;
            const int32_t kvplane = bnsd ? (w.seq * a.Hkv + kvh) : kvh;
            mbar_expect_tx(bar(C::kBarQFull), C::kTileBytes);
            for (int at = 0; at < C::kAtoms; ++at) {
                if (bnsd)
                    tma_load_3d(sbase + C::kOffQ + at * C::kAtomBytes, &tmQ, bar(C::kBarQFull), at * 64,
                                w.qt * kBlockM, qplane);
                else
                    tma_load_3d(sbase + C::kOffQ + at * C::kAtomBytes, &tmQ, bar(C::kBarQFull), at * 64, qplane,
                                w.tok0 + w.qt * kBlockM);
            }
            int32_t issued_k = 0, issued_v = 0;
            for (int32_t j = 0; j < n_kv; ++j) {
                const int s = j % C::kStages;
                const uint32_t u = static_cast<uint32_t>(j / C::kStages);
                if (u > 0 && !mbar_wait(bar(C::kBarKEmpty + s), (u - 1) & 1u, abort_flag)) break;
                mbar_expect_tx(bar(C::kBarKFull + s), C::kTileBytes);
                for (int at = 0; at < C::kAtoms; ++at) {
                    const uint32_t dst = sbase + C::kOffK + s * C::kTileBytes + at * C::kAtomBytes;
                    if (bnsd)
                        tma_load_3d(dst, &tmK, bar(C::kBarKFull + s), at * 64, j * kBlockN, kvplane);
                    else
                        tma_load_3d(dst, &tmK, bar(C::kBarKFull + s), at * 64, kvplane, w.tok0 + j * kBlockN);
                }
                issued_k = j + 1;
                if (u > 0 && !mbar_wait(bar(C::kBarVEmpty + s), (u - 1) & 1u, abort_flag)) break;
                mbar_expect_tx(bar(C::kBarVFull + s), C::kTileBytes);
                for (int at = 0; at < C::kAtoms; ++at) {
                    const uint32_t dst = sbase + C::kOffV + s * C::kTileBytes + at * C::kAtomBytes;
                    if (bnsd)
                        tma_load_3d(dst, &tmV, bar(C::kBarVFull + s), at * 64, j * kBlockN, kvplane);
                    else
                        tma_load_3d(dst, &tmV, bar(C::kBarVFull + s), at * 64, kvplane, w.tok0 + j * kBlockN);
                }
                issued_v = j + 1;
            }
            // Drain: every issued copy must have landed before the CTA exits.
            mbar_wait_drain(bar(C::kBarQFull), 0);
            for (int32_t j = (issued_k > C::kStages ? issued_k - C::kStages : 0); j < issued_k; ++j)
                mbar_wait_drain(bar(C::kBarKFull + j % C::kStages), static_cast<uint32_t>(j / C::kStages) & 1u);
            for (int32_t j = (issued_v > C::kStages ? issued_v - C::kStages : 0); j < issued_v; ++j)
                mbar_wait_drain(bar(C::kBarVFull + j % C::kStages), static_cast<uint32_t>(j / C::kStages) & 1u);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ tcgen05 issuer
        if (lane == 0) {
            constexpr uint32_t kIdescQK = idesc_f16(IoT<kFP16>::kFmt, 0, 0, kBlockM, kBlockN);
            constexpr uint32_t kIdescPV = idesc_f16(IoT<kFP16>::kFmt, 0, 1, kBlockM, D);
            bool ok = mbar_wait(bar(C::kBarQReady), 0, abort_flag);
            auto issue_pv = [&](int32_t i) -> bool {
                const int s = i % C::kStages;
                const uint32_t u = static_cast<uint32_t>(i / C::kStages);
                if (!mbar_wait(bar(C::kBarPFull), static_cast<uint32_t>(i) & 1u, abort_flag)) return false;
                if (!mbar_wait(bar(C::kBarVFull + s), u & 1u, abort_flag)) return false;
                tc_fence_after();
                const uint32_t vbase = sbase + C::kOffV + s * C::kTileBytes;
#pragma unroll
                for (int k = 0; k < kBlockN / 16; ++k) {
                    const uint64_t ad = smem_desc_sw128(sbase + C::kOffP + (k >> 2) * C::kAtomBytes + (k & 3) * 32,
                                                        16, 1024);
                    const uint64_t bd = smem_desc_sw128(vbase + k * 16 * 128, C::kAtomBytes, 1024);
                    umma_ss(tmem + C::kColO, ad, bd, kIdescPV, (i > 0 || k > 0) ? 1u : 0u);
                }
                tc_commit(bar(C::kBarPVDone));
                tc_commit(bar(C::kBarVEmpty + s));
                return true;
            };
            if (ok) {
                tc_fence_after();
                for (int32_t j = 0; j < n_kv && ok; ++j) {
                    const int s = j % C::kStages;
                    const uint32_t u = static_cast<uint32_t>(j / C::kStages);
                    const int b = j & 1;
                    if (!mbar_wait(bar(C::kBarKReady + s), u & 1u, abort_flag)) { ok = false; break; }
                    if (j >= 2 && !mbar_wait(bar(C::kBarSEmpty + b), static_cast<uint32_t>((j >> 1) - 1) & 1u,
                                             abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t kbase = sbase + C::kOffK + s * C::kTileBytes;
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t koff = (k >> 2) * C::kAtomBytes + (k & 3) * 32;
                        const uint64_t ad = smem_desc_sw128(sbase + C::kOffQ + koff, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(kbase + koff, 16, 1024);
                        umma_ss(tmem + C::kColS + b * kBlockN, ad, bd, kIdescQK, k > 0 ? 1u : 0u);
                    }
                    tc_commit(bar(C::kBarSFull + b));
                    tc_commit(bar(C::kBarKEmpty + s));
                    if (j >= 1) ok = issue_pv(j - 1);
                }
                if (ok) issue_pv(n_kv - 1);
            }
            tc_commit(bar(C::kBarMmaFin));
            mbar_wait_drain(bar(C::kBarMmaFin), 0);
        }
    } else if (warp >= kRopeWarp0) {
        // ------------------------------------------------------------ RoPE warpgroup
        const int32_t rt = threadIdx.x - kRopeWarp0 * 32;
        const float* table = a.table;
        if (mbar_wait(bar(C::kBarQFull), 0, abort_flag)) {
            const int32_t q0 = w.qt * kBlockM;
            rope_tile<D, kFP16>(sbase + C::kOffQ, min(kBlockM, w.L - q0),
                                table + static_cast<int64_t>(w.tok0 + q0) * D, rt);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarQReady));
            for (int32_t j = 0; j < n_kv; ++j) {
                const int s = j % C::kStages;
                const uint32_t u = static_cast<uint32_t>(j / C::kStages);
                if (!mbar_wait(bar(C::kBarKFull + s), u & 1u, abort_flag)) break;
                const int32_t k0 = j * kBlockN;
                rope_tile<D, kFP16>(sbase + C::kOffK + s * C::kTileBytes, min(kBlockN, w.L - k0),
                                    table + static_cast<int64_t>(w.tok0 + k0) * D, rt);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::kBarKReady + s));
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroup
        const int row = threadIdx.x;  // 0..127 == TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const int32_t qi = w.qt * kBlockM + row;
        const float sl2 = a.scale_log2;
        float m = -INFINITY;  // running max of score * scale * log2(e)
        float l = 0.0f;       // running sum of exp2(score * scale_log2 - m)
        bool ok = true;
        uint32_t sr[4][32];
        for (int32_t j = 0; j < n_kv; ++j) {
            const int b = j & 1;
            // tcgen05.ld/st are warp-collective: every decision below is warp-uniform.
            if (!__all_sync(0xffffffffu, mbar_wait(bar(C::kBarSFull + b), static_cast<uint32_t>(j >> 1) & 1u,
                                                   abort_flag))) { ok = false; break; }
            tc_fence_after();
            const uint32_t sc = tmem + lane_off + C::kColS + b * kBlockN;
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_ld32(sc + q * 32, sr[q]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarSEmpty + b));

            // mask: keys [kv0, kv0 + lim) are visible to this row
            const int32_t kv0 = j * kBlockN;
            const int32_t lim = (a.causal ? min(qi + 1, w.L) : w.L) - kv0;
            float mx = -INFINITY;
            if (lim >= kBlockN) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int c = 0; c < 32; ++c) mx = fmaxf(mx, __uint_as_float(sr[q][c]));
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        float v = (q * 32 + c < lim) ? __uint_as_float(sr[q][c]) : -INFINITY;
                        sr[q][c] = __float_as_uint(v);
                        mx = fmaxf(mx, v);
                    }
            }
            const float m_new = fmaxf(m, mx * sl2);
            if (j > 0) {
                // PV(j-1) must be done: it reads the P buffer and writes O.
                if (!__all_sync(0xffffffffu, mbar_wait(bar(C::kBarPVDone), static_cast<uint32_t>(j - 1) & 1u,
                                                       abort_flag))) { ok = false; break; }
                tc_fence_after();
                const bool need = m_new > m + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need)) {
                    const float alpha = need ? ex2(m - m_new) : 1.0f;
                    l *= alpha;
#pragma unroll 1
                    for (int q = 0; q < D / 32; ++q) {
                        uint32_t o[32];
                        tmem_ld32(tmem + lane_off + C::kColO + q * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                        tmem_st32(tmem + lane_off + C::kColO + q * 32, o);
                    }
                    tmem_wait_st();
                    if (need) m = m_new;
                }
            } else {
                m = m_new;
            }
            const float neg_m = (m == -INFINITY) ? 0.0f : -m;
            const uint32_t prow = sbase + C::kOffP + row * 128;
#pragma unroll
            for (int cc = 0; cc < kBlockN / 8; ++cc) {
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    p[e] = ex2(fmaf(__uint_as_float(sr[cc >> 2][(cc & 3) * 8 + e]), sl2, neg_m));
                    l += p[e];
                }
                uint4 v;
                v.x = IoT<kFP16>::pack(p[0], p[1]);
                v.y = IoT<kFP16>::pack(p[2], p[3]);
                v.z = IoT<kFP16>::pack(p[4], p[5]);
                v.w = IoT<kFP16>::pack(p[6], p[7]);
                sts128(prow + (cc >> 3) * C::kAtomBytes + (((cc & 7) ^ (row & 7)) << 4), v);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarPFull));
        }
        // epilogue: out = O / l
        const bool fin = ok && mbar_wait(bar(C::kBarPVDone), static_cast<uint32_t>(n_kv - 1) & 1u, abort_flag);
        if (__all_sync(0xffffffffu, fin)) {
            tc_fence_after();
            const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
            const bool valid = qi < w.L;
            using OutT = uint16_t;
            OutT* outp = reinterpret_cast<OutT*>(a.out);
            int64_t o_off;
            if (a.layout == 0)
                o_off = ((static_cast<int64_t>(w.seq) * a.Hq + w.h) * a.S + qi) * D;
            else
                o_off = (static_cast<int64_t>(w.tok0 + qi) * a.Hq + w.h) * D;
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + C::kColO + q * 32, o);
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
