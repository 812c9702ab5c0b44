// rope_sincos.cuh -- the DynamicNTK sin/cos table (page "DynamicNTKOperation",
// computation process: freq = outer(positionIds_b, invFreq_b),
// emb = cat(freq, freq), sin/cos of emb) and the compact cos/sin table that the
// fused attention kernel reads for its on-chip rotation.
//
// Both are HBM-write bound: one fp32 sincos per (token, frequency), each
// thread handles one token and 8 consecutive frequencies and writes 16-byte
// vectors.  The duplicated half of the public table reuses the same values, so
// columns j and j + D/2 are bit-identical by construction.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "sm100_ptx.cuh"
#include "stream_mem.cuh"

namespace rfa {

constexpr int kMaxSeqs = 16;     // page "DynamicNTKOperation", constraints: batch <= 16
constexpr int kMaxHalfHost = 64; // host-derived invFreq rows carried in kernel params (D <= 128)

template <typename T>
struct Pack8;  // 8 values -> the vector(s) stored for one chunk
template <>
struct Pack8<__half> {
    template <bool kStream>
    static __device__ __forceinline__ void store(__half* dst, const float (&v)[8]) {
        __half2 h[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) h[k] = __floats2half2_rn(v[2 * k], v[2 * k + 1]);
        stg128<kStream>(dst, *reinterpret_cast<uint4*>(h));
    }
};
template <>
struct Pack8<__nv_bfloat16> {
    template <bool kStream>
    static __device__ __forceinline__ void store(__nv_bfloat16* dst, const float (&v)[8]) {
        __nv_bfloat162 h[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) h[k] = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
        stg128<kStream>(dst, *reinterpret_cast<uint4*>(h));
    }
};
template <>
struct Pack8<float> {
    template <bool kStream>
    static __device__ __forceinline__ void store(float* dst, const float (&v)[8]) {
        stg128<kStream>(dst, make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                                        __float_as_uint(v[3])));
        stg128<kStream>(dst + 4, make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]),
                                            __float_as_uint(v[7])));
    }
};

// sin/cos of the angles position * invFreq[j], j = j0 .. j0+7.
// The fp32 product x = p * w is reduced by 2*pi with the two-constant
// Cody-Waite scheme (W. J. Cody and W. Waite, "Software Manual for the
// Elementary Functions", 1980): k = round(x / 2pi), r = (x - k C1) - k C2 with
// C1 + C2 = 2pi to ~7e-15 (both products exact inside fma).  The rounding error
// of x itself, recovered exactly as fma(p, w, -x), is added back to r, so the
// angle carries no error from the fp32 product.  The SFU then evaluates sin and
// cos of r, which lies in [-pi, pi] up to a few ulps for |x| below ~1e6 (beyond
// that the quotient's rounding can leave |r| a few multiples of 2pi larger, still
// within the SFU's accurate range for the 16-bit outputs).
constexpr float kTwoPiHi = 6.2831854820251465f;      // fp32 nearest to 2 pi
constexpr float kTwoPiLo = -1.7484555314695172e-07f;  // 2 pi - kTwoPiHi, rounded to fp32
constexpr float kInvTwoPi = 0.15915493667125702f;     // fp32 nearest to 1 / (2 pi)
__device__ __forceinline__ void sincos_reduced(float p, float w, float& s, float& c) {
    const float x = p * w;
    const float xe = fmaf(p, w, -x);  // p * w - x, exactly
    const float k = rintf(x * kInvTwoPi);
    const float r = fmaf(-k, kTwoPiLo, fmaf(-k, kTwoPiHi, x)) + xe;
    __sincosf(r, &s, &c);
}

__device__ __forceinline__ void sincos8(float position, const float* inv, float (&s)[8], float (&c)[8]) {
    // Generic loads: `inv` points either to global memory or into the
    // kernel's parameter block (host-derived frequencies).
    const float4 i0 = reinterpret_cast<const float4*>(inv)[0];
    const float4 i1 = reinterpret_cast<const float4*>(inv)[1];
    const float iv[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) sincos_reduced(position, iv[k], s[k], c[k]);
}

// Public table: sin/cos [ntokens, headSize] from device positions, invFreq
// [batch, headSize/2] and device seqLens [batch].  kStream: the stores carry
// the evict-first hint (the host sets it when the two tables exceed half of L2;
// measured on 131 MB of fp16 tables, back to back: 4.86 -> 5.28 TB/s).
template <typename OutT, bool kStream>
__global__ void __launch_bounds__(256) rope_sincos_kernel(const int32_t* __restrict__ pos,
                                                          const float* __restrict__ inv,
                                                          const int32_t* __restrict__ seqLens, int32_t batch,
                                                          int32_t ntokens, int32_t headSize, OutT* __restrict__ sinOut,
                                                          OutT* __restrict__ cosOut) {
    __shared__ int32_t s_cum[kMaxSeqs + 1];
    __shared__ int32_t s_ok;
    if (threadIdx.x < 32) {
        // prefix sums of the lengths: one load per lane, then a warp scan
        const int32_t lane = threadIdx.x;
        const int64_t L = (lane < batch) ? static_cast<int64_t>(__ldg(seqLens + lane)) : 0;
        int64_t x = L;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        const bool bad = __any_sync(0xffffffffu, lane < batch && L <= 0);
        const int64_t total = __shfl_sync(0xffffffffu, x, batch - 1);
        if (lane < batch) s_cum[lane + 1] = static_cast<int32_t>(x);
        if (lane == 0) {
            s_cum[0] = 0;
            const int32_t ok = (!bad && total == ntokens) ? 1 : 0;
            s_ok = ok;
            if (!ok && blockIdx.x == 0) record_status(1 /* RFA_ERR_INVALID_ARG */);
        }
    }
    __syncthreads();
    if (!s_ok) return;
    const int32_t half = headSize >> 1;
    const uint32_t chunks = static_cast<uint32_t>(half >> 3);
    // ntokens <= 256000 and chunks <= 128: the work index fits 32 bits
    const uint32_t work = static_cast<uint32_t>(ntokens) * chunks;
    for (uint32_t w = blockIdx.x * blockDim.x + threadIdx.x; w < work; w += gridDim.x * blockDim.x) {
        const int32_t t = static_cast<int32_t>(w / chunks);
        const int32_t c = static_cast<int32_t>(w - static_cast<uint32_t>(t) * chunks);
        // segment of token t: the last b with s_cum[b] <= t (binary search over at most 16)
        int32_t b = 0;
#pragma unroll
        for (int step = kMaxSeqs / 2; step > 0; step >>= 1)
            if (b + step < batch && t >= s_cum[b + step]) b += step;
        const int64_t o = static_cast<int64_t>(t) * headSize + 8 * c;
        if (!in_bounds(t < ntokens && b < batch && 8 * c + 8 <= half &&
                       o + half + 8 <= static_cast<int64_t>(ntokens) * headSize))
            continue;
        float s[8], co[8];
        sincos8(static_cast<float>(__ldg(pos + t)), inv + static_cast<int64_t>(b) * half + 8 * c, s, co);
        Pack8<OutT>::template store<kStream>(sinOut + o, s);
        Pack8<OutT>::template store<kStream>(sinOut + o + half, s);
        Pack8<OutT>::template store<kStream>(cosOut + o, co);
        Pack8<OutT>::template store<kStream>(cosOut + o + half, co);
    }
}

// Compact table for the fused kernel.  Per token, 16-byte chunks cover 4
// frequencies j0..j0+3 as four 32-bit words of fp16 pairs:
//   (cos j0, cos j0+1), (sin j0, sin j0+1), (cos j0+2, cos j0+3), (sin j0+2, sin j0+3)
// so that one conversion yields the packed fp32 operands of two dimensions.
// Chunk order within a row: for half == 64 the chunk of frequency group
// g = j0/4 is stored at position (g % 2) * 8 + g / 2, so the fused kernel's 8
// lanes that share a row read distinct shared-memory banks; for other sizes
// the order is natural.  Segments: uniform_len > 0 -> segment t / uniform_len,
// otherwise the host-known prefix sums cum[].
// Per-sequence seeds of the fused kernel's in-tile angle recurrence, used when
// a sequence's positions are consecutive (pos[tok0 + i] == pos[tok0] + i): a
// RoPE thread forms the angles (P + row) w_j of its first row of a tile
// directly (fp64 angle reduced modulo 2 pi, then sin/cos), and reaches its
// other rows of the tile, `step` rows apart, by complex multiplication with
// wstep_j = (cos, sin)(step w_j), step = 1024 / (D/2) rows (the RoPE threads
// sharing a row column).  wstep is evaluated in fp64 and rounded once to fp32.
struct RopeSeed {
    int32_t consecutive;  // 1: the recurrence applies to this sequence
    int32_t pos0;         // P
    int32_t pad[2];
    float2 wstep[kMaxHalfHost];  // (cos, sin) of step * w_j
    float inv[kMaxHalfHost];     // w_j
};

struct TableArgs {
    const int32_t* pos;
    const float* inv_dev;  // [nseg, half] or nullptr -> inv_host
    uint32_t* table;       // [ntokens][half] 32-bit words of fp16 cos/sin pairs
    RopeSeed* seeds;       // [nseg]
    int32_t* sched;        // the fused kernel's work counters [0..1] (zeroed here) and, at [2], the
                           // launch flag "every sequence's positions are consecutive", or nullptr
    int32_t npos;          // entries of pos
    int32_t inv_dev_rows;  // rows of inv_dev
    int32_t ntokens;
    int32_t half;
    int32_t nseg;
    int32_t uniform_len;
    int32_t inv_host_rows;  // 1: one row shared by all segments; else one per segment
    int32_t pos_sq;         // > 0: row t reads pos[(t / uniform_len) * pos_sq + t % pos_sq] (decode query rows)
    int32_t cum[kMaxSeqs + 1];
    alignas(16) float inv_host[kMaxSeqs * kMaxHalfHost];
};

__global__ void __launch_bounds__(256) rope_table_kernel(const __grid_constant__ TableArgs a) {
    // the attention launch that follows on the stream starts from zeroed work counters
    if (a.sched != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
        a.sched[0] = 0;
        a.sched[1] = 0;
    }
    const int32_t chunks = a.half >> 3;
    const int64_t work = static_cast<int64_t>(a.ntokens) * chunks;
    for (int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; w < work;
         w += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int32_t t = static_cast<int32_t>(w / chunks);
        const int32_t c = static_cast<int32_t>(w - static_cast<int64_t>(t) * chunks);
        int32_t b;
        if (a.uniform_len > 0) {
            b = t / a.uniform_len;
        } else {
            b = 0;
            while (b + 1 < a.nseg && t >= a.cum[b + 1]) ++b;
        }
        const float* inv = a.inv_dev ? a.inv_dev + static_cast<int64_t>(b) * a.half
                                     : a.inv_host + (a.inv_host_rows == 1 ? 0 : b) * a.half;
        float s[8], co[8];
        const int32_t pt = a.pos_sq > 0 ? (t / a.uniform_len) * a.pos_sq + t % a.pos_sq : t;
        const int g0 = (a.half == 64) ? c : 2 * c;
        const int g1 = (a.half == 64) ? 8 + c : 2 * c + 1;
        const bool inv_ok = a.inv_dev ? (b < a.inv_dev_rows) : (a.inv_host_rows == 1 || b < a.inv_host_rows);
        if (!in_bounds(pt >= 0 && pt < a.npos && b >= 0 && inv_ok && 8 * c + 8 <= a.half && g0 < a.half / 4 &&
                       g1 < a.half / 4))
            continue;
        const int32_t p = __ldg(a.pos + pt);
        sincos8(static_cast<float>(p), inv + 8 * c, s, co);
        if (a.seeds != nullptr && c == 0) {
            // a position that breaks the sequence's run (compared in 64 bits, so positions wrapping
            // past INT32_MAX do not count as consecutive) clears its consecutive flag, which
            // rope_seed_kernel set before this kernel
            const int32_t tok0 = a.uniform_len > 0 ? b * a.uniform_len : a.cum[b];
            if (static_cast<int64_t>(p) != static_cast<int64_t>(__ldg(a.pos + tok0)) + (t - tok0)) {
                a.seeds[b].consecutive = 0;
                if (a.sched != nullptr) a.sched[2] = 0;
            }
        }
        uint32_t pr[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            __half2 hc = __floats2half2_rn(co[2 * k], co[2 * k + 1]);
            __half2 hs = __floats2half2_rn(s[2 * k], s[2 * k + 1]);
            pr[2 * k] = *reinterpret_cast<uint32_t*>(&hc);
            pr[2 * k + 1] = *reinterpret_cast<uint32_t*>(&hs);
        }
        uint4* row = reinterpret_cast<uint4*>(a.table + static_cast<int64_t>(t) * a.half);
        // groups 2c and 2c+1 of 4 pairs each
        row[g0] = make_uint4(pr[0], pr[1], pr[2], pr[3]);
        row[g1] = make_uint4(pr[4], pr[5], pr[6], pr[7]);
    }
}

// Per-sequence seeds (grid: one block per sequence; runs before
// rope_table_kernel, which clears the consecutive flag of a sequence whose
// positions break the run, and the launch-wide flag with it): the flags set,
// the first position, the invFreq row
// and the in-tile step (cos, sin) of step * w_j, the angle formed and reduced
// modulo 2 pi in fp64, then evaluated with fp32 sincos (|error| ~1e-7).
__global__ void __launch_bounds__(64) rope_seed_kernel(const __grid_constant__ TableArgs a) {
    const int32_t b = blockIdx.x;
    const int32_t tok0 = a.uniform_len > 0 ? b * a.uniform_len : a.cum[b];
    if (!in_bounds(b < a.nseg && tok0 >= 0 && tok0 < a.ntokens && tok0 < a.npos)) return;
    RopeSeed* sd = a.seeds + b;
    if (threadIdx.x == 0) {
        sd->consecutive = 1;
        sd->pos0 = __ldg(a.pos + tok0);
        if (b == 0 && a.sched != nullptr) a.sched[2] = 1;  // cleared by rope_table_kernel on any break
    }
    const float* inv = a.inv_dev ? a.inv_dev + static_cast<int64_t>(b) * a.half
                                 : a.inv_host + (a.inv_host_rows == 1 ? 0 : b) * a.half;
    const double two_pi = 6.283185307179586476925286766559;
    const double step = 1024.0 / static_cast<double>(a.half);  // rows between a RoPE thread's rows
    for (int32_t j = threadIdx.x; j < a.half; j += blockDim.x) {
        const double w = static_cast<double>(inv[j]);
        double ang = step * w;
        ang -= two_pi * rint(ang / two_pi);
        float sn, cs;
        sincosf(static_cast<float>(ang), &sn, &cs);
        sd->wstep[j] = make_float2(cs, sn);
        sd->inv[j] = inv[j];
    }
}

}  // namespace rfa
