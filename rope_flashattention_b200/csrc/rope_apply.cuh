// rope_apply.cuh -- the Rope operator: q, k and their tokens' sin/cos table
// rows in, rotated q and k out (page "DynamicNTKOperation", operator context:
// DynamicNTK's sin and cos go with q and k into the Rope operator), with an
// optional write of the rotated keys into a KV cache.
//
//   out[j] = x[j] * cos[j] + rot(x)[j] * sin[j]
//   rotate-half pairs: rot(x) = (-x[D/2..D), x[0..D/2))
//   adjacent pairs (page "RoPE, RMSNorm, GQA/MQA, SwiGLU, MoE", sec. 6):
//                      rot(x)[2i] = -x[2i+1], rot(x)[2i+1] = x[2i]
//
// HBM-bound elementwise work.  A thread owns one token row, one 8-element
// chunk in each half of D (elements 8c.. and D/2 + 8c..) and a group of up to
// kApplyHeads heads: it reads its 2 x 8 cos and sin values once, then rotates
// that chunk pair of each head with 16-byte loads and stores.  Eight
// consecutive threads cover one 256-byte row (D = 128), so accesses coalesce.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "sm100_ptx.cuh"
#include "stream_mem.cuh"

namespace rfa {

constexpr int kApplyHeads = 8;  // heads per thread
constexpr int kApplyBatch = 4;  // heads whose loads are in flight together

struct RopeApplyArgs {
    const void* q;
    const void* k;
    const void* sin_t;
    const void* cos_t;
    void* q_out;
    void* k_out;
    const int32_t* slots;  // [R] or nullptr
    void* cache;           // [cache_rows, Hkv, D] or nullptr
    int64_t cache_rows;
    int32_t bnsd;          // 1: x [B, H, S, D]; 0: x [R, H, D]
    int32_t R;             // token rows (T, or B * S)
    int32_t S;             // BNSD sequence length
    int32_t Hq, Hkv, D;
};

// 8 consecutive table values as fp32
template <typename TabT>
struct Tab8;
template <>
struct Tab8<__half> {
    static __device__ __forceinline__ void load(const void* p, float (&v)[8]) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
};
template <>
struct Tab8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const void* p, float (&v)[8]) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};
template <>
struct Tab8<float> {
    static __device__ __forceinline__ void load(const void* p, float (&v)[8]) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(p));
        const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

// 8 bf16 / fp16 values <-> fp32
template <bool kFP16>
__device__ __forceinline__ void unpack8(const uint4& u, float (&v)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if constexpr (kFP16) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        } else {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
}
template <bool kFP16>
__device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if constexpr (kFP16) {
            const __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&h);
        } else {
            const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// kStream: q/k loads and all stores carry the evict-first hint (stream_mem.cuh).
template <bool kFP16, typename TabT, bool kInterleaved, bool kStream>
__global__ void __launch_bounds__(256) rope_apply_kernel(const RopeApplyArgs a) {
    const uint32_t chunks = static_cast<uint32_t>(a.D) / 16u;  // chunk pairs per row
    const int32_t H = a.Hq + a.Hkv;
    const uint32_t hgroups = static_cast<uint32_t>((H + kApplyHeads - 1) / kApplyHeads);
    const uint32_t work = static_cast<uint32_t>(a.R) * hgroups * chunks;  // < 2^31, checked on the host
    const int32_t half = a.D / 2;
    for (uint32_t w = blockIdx.x * blockDim.x + threadIdx.x; w < work; w += gridDim.x * blockDim.x) {
        const uint32_t c = w % chunks;
        const uint32_t rem = w / chunks;
        const int32_t hg = static_cast<int32_t>(rem % hgroups);
        const int32_t r = static_cast<int32_t>(rem / hgroups);
        const int32_t e0 = 8 * static_cast<int32_t>(c), e1 = half + e0;
        // every row index below derives from r < R and a head < Hq + Hkv
        if (!in_bounds(r >= 0 && r < a.R && hg * kApplyHeads < H && e1 + 8 <= a.D)) continue;
        const size_t tsz = sizeof(TabT);
        const char* srow = static_cast<const char*>(a.sin_t) + static_cast<size_t>(r) * a.D * tsz;
        const char* crow = static_cast<const char*>(a.cos_t) + static_cast<size_t>(r) * a.D * tsz;
        float s0[8], s1[8], c0[8], c1[8];
        Tab8<TabT>::load(srow + e0 * tsz, s0);
        Tab8<TabT>::load(srow + e1 * tsz, s1);
        Tab8<TabT>::load(crow + e0 * tsz, c0);
        Tab8<TabT>::load(crow + e1 * tsz, c1);
        const int32_t h0 = hg * kApplyHeads;
        const int32_t h1 = min(h0 + kApplyHeads, H);
        int32_t slot = -1;
        if (a.slots != nullptr && h1 > a.Hq) slot = __ldg(a.slots + r);
        const int32_t b = a.bnsd ? r / a.S : 0, s = a.bnsd ? r - b * a.S : 0;
        auto row_of = [&](int32_t h, bool& is_k, int32_t& hx) -> int64_t {
            is_k = h >= a.Hq;
            hx = is_k ? h - a.Hq : h;
            const int32_t Hx = is_k ? a.Hkv : a.Hq;
            return a.bnsd ? (static_cast<int64_t>(b) * Hx + hx) * a.S + s : static_cast<int64_t>(r) * Hx + hx;
        };
        // Heads in batches of kApplyBatch: every load of a batch is issued before its first
        // store, so each thread keeps kApplyBatch x 32 bytes in flight (the outputs may alias
        // the inputs, which stops the compiler from hoisting loads above stores itself).
#pragma unroll 1
        for (int32_t hb = h0; hb < h1; hb += kApplyBatch) {
            uint4 xa[kApplyBatch], xb[kApplyBatch];
#pragma unroll
            for (int u = 0; u < kApplyBatch; ++u) {
                if (hb + u < h1) {
                    bool is_k;
                    int32_t hx;
                    const int64_t row = row_of(hb + u, is_k, hx);
                    const uint16_t* src = static_cast<const uint16_t*>(is_k ? a.k : a.q) + row * a.D;
                    xa[u] = ldg128<kStream>(src + e0);
                    xb[u] = ldg128<kStream>(src + e1);
                }
            }
#pragma unroll
            for (int u = 0; u < kApplyBatch; ++u) {
                if (hb + u >= h1) break;
                bool is_k;
                int32_t hx;
                const int64_t row = row_of(hb + u, is_k, hx);
                float x0[8], x1[8], o0[8], o1[8];
                unpack8<kFP16>(xa[u], x0);
                unpack8<kFP16>(xb[u], x1);
                if constexpr (kInterleaved) {
#pragma unroll
                    for (int i = 0; i < 8; i += 2) {
                        o0[i] = fmaf(x0[i], c0[i], -x0[i + 1] * s0[i]);
                        o0[i + 1] = fmaf(x0[i + 1], c0[i + 1], x0[i] * s0[i + 1]);
                        o1[i] = fmaf(x1[i], c1[i], -x1[i + 1] * s1[i]);
                        o1[i + 1] = fmaf(x1[i + 1], c1[i + 1], x1[i] * s1[i + 1]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        o0[i] = fmaf(x0[i], c0[i], -x1[i] * s0[i]);
                        o1[i] = fmaf(x1[i], c1[i], x0[i] * s1[i]);
                    }
                }
                const uint4 p0 = pack8<kFP16>(o0), p1 = pack8<kFP16>(o1);
                void* dst = is_k ? a.k_out : a.q_out;
                if (dst != nullptr) {
                    uint16_t* d = static_cast<uint16_t*>(dst) + row * a.D;
                    stg128<kStream>(d + e0, p0);
                    stg128<kStream>(d + e1, p1);
                }
                if (is_k && slot >= 0) {
                    if (slot < a.cache_rows) {
                        uint16_t* d = static_cast<uint16_t*>(a.cache) + (static_cast<int64_t>(slot) * a.Hkv + hx) * a.D;
                        stg128<kStream>(d + e0, p0);
                        stg128<kStream>(d + e1, p1);
                    } else {
                        record_status(1 /* RFA_ERR_INVALID_ARG */);
                    }
                }
            }
        }
    }
}

// RMSNorm + RoPE + KV-cache write (the kv_rms_norm_rope_cache op named on page
// "RoPE fused into attention on Ascend", sec. 5.2; RMSNorm from page "RoPE,
// RMSNorm, GQA/MQA, SwiGLU, MoE", sec. 8): for token t and kv head h,
//   k_cache[slot_t, h] = rope(gamma * k[t,h] / sqrt(mean(k[t,h]^2) + eps))
//   v_cache[slot_t, h] = v[t,h]
// slots < 0 are skipped.  Same thread layout as rope_apply_kernel (one thread
// per row and chunk pair); a row's D/16 threads are consecutive lanes of one
// warp and sum their squares with shuffles, so D/16 must be a power of two
// dividing 32.  The grid-stride loop advances whole warps: every lane of a
// warp runs the same iterations (lanes past the end carry zeros).
struct KvCacheArgs {
    const void* k;
    const void* v;
    const float* gamma;
    const void* sin_t;
    const void* cos_t;
    const int32_t* slots;
    void* k_cache;
    void* v_cache;
    int64_t cache_rows;
    int32_t T, Hkv, D;
    float eps;
};

// kStream: k/v loads and the cache stores carry the evict-first hint (stream_mem.cuh).
template <bool kFP16, typename TabT, bool kInterleaved, bool kStream>
__global__ void __launch_bounds__(256, 4) kv_norm_rope_cache_kernel(const KvCacheArgs a) {
    const uint32_t chunks = static_cast<uint32_t>(a.D) / 16u;  // power of two <= 32
    const uint32_t work = static_cast<uint32_t>(a.T) * static_cast<uint32_t>(a.Hkv) * chunks;
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t stride = gridDim.x * blockDim.x;
    const int32_t half = a.D / 2;
    for (uint32_t base = blockIdx.x * blockDim.x + (threadIdx.x & ~31u); base < work; base += stride) {
        const uint32_t w = base + lane;
        const bool act = w < work;
        const uint32_t c = w % chunks;
        const uint32_t row = w / chunks;  // t * Hkv + h
        const int32_t t = act ? static_cast<int32_t>(row / static_cast<uint32_t>(a.Hkv)) : 0;
        const int32_t h = act ? static_cast<int32_t>(row - static_cast<uint32_t>(t) * a.Hkv) : 0;
        const int32_t e0 = 8 * static_cast<int32_t>(c), e1 = half + e0;
        const int64_t off = (static_cast<int64_t>(t) * a.Hkv + h) * a.D;
        const bool in_range = !act || in_bounds(t < a.T && h < a.Hkv && e1 + 8 <= a.D);
        // k, v and the slot are loaded together, before any store of this iteration (the
        // caches do not overlap k and v), so their latencies overlap
        uint4 ka = make_uint4(0u, 0u, 0u, 0u), kb = ka, va = ka, vb = ka;
        int32_t slot = -1;
        if (act && in_range) {
            const uint16_t* src = static_cast<const uint16_t*>(a.k) + off;
            const uint16_t* vs = static_cast<const uint16_t*>(a.v) + off;
            ka = ldg128<kStream>(src + e0);
            kb = ldg128<kStream>(src + e1);
            va = ldg128<kStream>(vs + e0);
            vb = ldg128<kStream>(vs + e1);
            slot = __ldg(a.slots + t);
        }
        float x0[8], x1[8];
        unpack8<kFP16>(ka, x0);
        unpack8<kFP16>(kb, x1);
        float ss = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(x0[i], x0[i], fmaf(x1[i], x1[i], ss));
        for (uint32_t o = chunks >> 1; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (!act || !in_range || slot < 0) continue;
        if (slot >= a.cache_rows) {
            record_status(1 /* RFA_ERR_INVALID_ARG */);
            continue;
        }
        const float inv = rsqrtf(ss / static_cast<float>(a.D) + a.eps);
        float g0[8], g1[8];
        Tab8<float>::load(a.gamma + e0, g0);
        Tab8<float>::load(a.gamma + e1, g1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            x0[i] = g0[i] * (x0[i] * inv);
            x1[i] = g1[i] * (x1[i] * inv);
        }
        const size_t tsz = sizeof(TabT);
        const char* srow = static_cast<const char*>(a.sin_t) + static_cast<size_t>(t) * a.D * tsz;
        const char* crow = static_cast<const char*>(a.cos_t) + static_cast<size_t>(t) * a.D * tsz;
        float s0[8], s1[8], c0[8], c1[8], o0[8], o1[8];
        Tab8<TabT>::load(srow + e0 * tsz, s0);
        Tab8<TabT>::load(srow + e1 * tsz, s1);
        Tab8<TabT>::load(crow + e0 * tsz, c0);
        Tab8<TabT>::load(crow + e1 * tsz, c1);
        if constexpr (kInterleaved) {
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                o0[i] = fmaf(x0[i], c0[i], -x0[i + 1] * s0[i]);
                o0[i + 1] = fmaf(x0[i + 1], c0[i + 1], x0[i] * s0[i + 1]);
                o1[i] = fmaf(x1[i], c1[i], -x1[i + 1] * s1[i]);
                o1[i + 1] = fmaf(x1[i + 1], c1[i + 1], x1[i] * s1[i + 1]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                o0[i] = fmaf(x0[i], c0[i], -x1[i] * s0[i]);
                o1[i] = fmaf(x1[i], c1[i], x0[i] * s1[i]);
            }
        }
        const int64_t dst = (static_cast<int64_t>(slot) * a.Hkv + h) * a.D;
        uint16_t* kd = static_cast<uint16_t*>(a.k_cache) + dst;
        stg128<kStream>(kd + e0, pack8<kFP16>(o0));
        stg128<kStream>(kd + e1, pack8<kFP16>(o1));
        uint16_t* vd = static_cast<uint16_t*>(a.v_cache) + dst;
        stg128<kStream>(vd + e0, va);
        stg128<kStream>(vd + e1, vb);
    }
}

}  // namespace rfa
