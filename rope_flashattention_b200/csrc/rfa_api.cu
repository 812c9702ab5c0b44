// rfa_api.cu -- the C ABI of librfa.so (declared in include/rfa.h): host-side
// validation, inverse frequencies (fp64 on the host, rounded once to fp32),
// work decomposition, TMA tensor maps and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "fused_rope_attn.cuh"
#include "rfa.h"
#include "rope_apply.cuh"
#include "rope_sincos.cuh"

namespace {

constexpr int32_t kVersion = 100;  // 0.1.0
constexpr int kMaxDevices = 64;

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3-D bf16/fp16 tensor map, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, bool fp16, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t st1,
              uint64_t st2, uint32_t b0, uint32_t b1, uint32_t b2) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {st1, st2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                    const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Opt-in to large dynamic shared memory, once per (kernel, device).  The
// template tag keeps one flag set per kernel instantiation.
// The cos/sin table as a 3-D map of 32-bit (cos, sin) pairs: [1][T][D/2],
// boxes of 32 pairs (128 B) x 128 tokens, 128-byte swizzle.
bool make_table_map(CUtensorMap* m, const void* base, uint64_t T, int D) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D / 2), T, 1};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D / 2) * 4, T * (D / 2) * 4};
    cuuint32_t box[3] = {32, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int kTag, typename K>
rfa_status ensure_smem_attr(K kernel, int bytes) {
    static bool done[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RFA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(mu);
    if (!done[dev]) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
            return RFA_ERR_CUDA;
        done[dev] = true;
    }
    return RFA_OK;
}

int grid_for(int64_t work, int threads) {
    int64_t blocks = (work + threads - 1) / threads;
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(blocks, 148LL * 64)));
}

// SMs of the current device; 148 (a B200) when no device is visible, so that
// host-only planning (workspace sizes) matches the GPU it is meant for.
int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
        (void)cudaGetLastError();  // not a launch error: leave no error behind
        return 148;
    }
    return sms;
}

// Grid of a grid-stride kernel: no more blocks than fit on the device at once
// (every block then pays its prologue once).
template <typename K>
int resident_grid(K kernel, int64_t work, int threads) {
    const int sms = device_sms();
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess || per_sm < 1) {
        (void)cudaGetLastError();
        per_sm = 1;
    }
    const int64_t blocks = (work + threads - 1) / threads;
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(blocks, static_cast<int64_t>(sms) * per_sm)));
}

// L2 size of the current device in bytes; 126 MB (a B200) when no device is visible.
int64_t device_l2_bytes() {
    int dev = 0, l2 = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess ||
        l2 < 1) {
        (void)cudaGetLastError();
        return 126ll << 20;
    }
    return l2;
}

// True when a launch moving `bytes` should use the evict-first accesses of stream_mem.cuh.
bool streams(double bytes) { return bytes > 0.5 * static_cast<double>(device_l2_bytes()); }

// The public sin/cos table kernel; stream_out selects its evict-first stores.
template <typename OutT>
void launch_sincos(bool stream_out, int64_t work, cudaStream_t st, const int32_t* pos, const float* inv,
                   const int32_t* lens, int32_t batch, int32_t ntokens, int32_t headSize, void* sinOut, void* cosOut) {
    auto k = stream_out ? rfa::rope_sincos_kernel<OutT, true> : rfa::rope_sincos_kernel<OutT, false>;
    k<<<resident_grid(k, work, 256), 256, 0, st>>>(pos, inv, lens, batch, ntokens, headSize, static_cast<OutT*>(sinOut),
                                                   static_cast<OutT*>(cosOut));
}

// invFreq_j = base^(-2j/D) in fp64, rounded once to fp32.
void inv_freq_row(double base, int D, float* out) {
    for (int j = 0; j < D / 2; ++j) out[j] = static_cast<float>(std::pow(base, -2.0 * j / static_cast<double>(D)));
}

double ntk_base(const rfa_attn_params* p, int64_t S_b) {
    if (!p->ntk_enable || S_b <= p->ntk_train_len) return p->rope_base;
    const double f = p->ntk_factor;
    return p->rope_base * std::pow(f * static_cast<double>(S_b) / p->ntk_train_len - (f - 1.0),
                                   static_cast<double>(p->D) / (p->D - 2));
}

rfa_status validate_attn(const rfa_attn_params* p) {
    if (!p) return RFA_ERR_INVALID_ARG;
    if (p->layout != RFA_LAYOUT_BNSD && p->layout != RFA_LAYOUT_TND) return RFA_ERR_INVALID_ARG;
    if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->D < 1) return RFA_ERR_INVALID_ARG;
    if (p->Hq % p->Hkv != 0) return RFA_ERR_INVALID_ARG;
    if (p->layout == RFA_LAYOUT_BNSD && p->S < 1) return RFA_ERR_INVALID_ARG;
    if (p->layout == RFA_LAYOUT_TND && p->B > rfa::kMaxSeqs) return RFA_ERR_INVALID_ARG;
    if (p->io_dtype != RFA_DT_BF16 && p->io_dtype != RFA_DT_FP16) {
        return p->io_dtype == RFA_DT_UNDEFINED ? RFA_ERR_INVALID_ARG : RFA_ERR_UNSUPPORTED;
    }
    if (!(p->scale >= 0.0f) || !std::isfinite(p->scale)) return RFA_ERR_INVALID_ARG;
    if (!(p->rope_base > 0.0) || !std::isfinite(p->rope_base)) return RFA_ERR_INVALID_ARG;
    if (p->ntk_enable && (p->ntk_train_len < 1 || !(p->ntk_factor >= 1.0) || !std::isfinite(p->ntk_factor)))
        return RFA_ERR_INVALID_ARG;
    if ((p->D & 1) != 0) return RFA_ERR_INVALID_ARG;
    if (p->rope_interleaved != 0 && p->rope_interleaved != 1) return RFA_ERR_INVALID_ARG;
    if (p->D != 64 && p->D != 128) return RFA_ERR_UNSUPPORTED;
    return RFA_OK;
}

int64_t total_tokens(const rfa_attn_params* p, const int32_t* lens) {
    if (p->layout == RFA_LAYOUT_BNSD) return static_cast<int64_t>(p->B) * p->S;
    int64_t t = 0;
    for (int b = 0; b < p->B; ++b) t += lens[b];
    return t;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// cos/sin table (D/2 fp16 cos and D/2 fp16 sin values per token), then one
// recurrence seed block per sequence, then the attention kernel's two work
// counters (zeroed by the table kernel, re-zeroed by the attention kernel's
// last CTA).
size_t table_bytes(int64_t T, int D) { return round_up(static_cast<size_t>(T) * D * 2, 256); }
size_t seeds_bytes(int nseg) { return round_up(static_cast<size_t>(nseg) * sizeof(rfa::RopeSeed), 256); }
constexpr size_t kSchedBytes = 256;
size_t workspace_bytes(int64_t T, int D, int nseg) { return table_bytes(T, D) + seeds_bytes(nseg) + kSchedBytes; }
int32_t* sched_of(void* workspace, int64_t T, int D, int nseg) {
    return reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + table_bytes(T, D) + seeds_bytes(nseg));
}

// Prefill: a persistent grid, one CTA per SM (one fits: 24 warps, ~226 KB of
// shared memory), each taking items from the work counters; decode: one CTA
// per item.
template <int D, bool kFP16, bool kAdj, bool kDecode = false>
rfa_status launch_attn(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mt,
                       const CUtensorMap& mo, const rfa::AttnArgs& args, cudaStream_t st) {
    auto kern = rfa::fused_rope_attn_fwd_kernel<D, kFP16, kAdj, kDecode>;
    constexpr int smem = rfa::AttnCfg<D>::kSmemBytes;
    constexpr int kTag = ((D * 4 + (kFP16 ? 2 : 0) + (kAdj ? 1 : 0)) << 1) + (kDecode ? 1 : 0);
    if (ensure_smem_attr<kTag>(kern, smem) != RFA_OK) return RFA_ERR_CUDA;
    const int grid = kDecode ? args.n_items : std::max(1, std::min(args.n_items, device_sms()));
    kern<<<grid, rfa::kAttnThreads, smem, st>>>(mq, mk, mv, mt, mo, args);
    return cudaGetLastError() == cudaSuccess ? RFA_OK : RFA_ERR_CUDA;
}

}  // namespace

extern "C" {

int32_t rfa_version(void) { return kVersion; }

const char* rfa_status_string(rfa_status s) {
    switch (s) {
        case RFA_OK: return "RFA_OK";
        case RFA_ERR_INVALID_ARG: return "RFA_ERR_INVALID_ARG";
        case RFA_ERR_UNSUPPORTED: return "RFA_ERR_UNSUPPORTED";
        case RFA_ERR_WORKSPACE: return "RFA_ERR_WORKSPACE";
        case RFA_ERR_CUDA: return "RFA_ERR_CUDA";
        case RFA_ERR_TIMEOUT: return "RFA_ERR_TIMEOUT";
    }
    return "RFA_ERR_UNKNOWN";
}

rfa_status rfa_get_device_status(void* stream) {
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return RFA_ERR_CUDA;
    int32_t v = 0;
    if (cudaMemcpyFromSymbol(&v, rfa::g_status, sizeof v) != cudaSuccess) return RFA_ERR_CUDA;
    const int32_t zero = 0;
    if (cudaMemcpyToSymbol(rfa::g_status, &zero, sizeof zero) != cudaSuccess) return RFA_ERR_CUDA;
    return static_cast<rfa_status>(v);
}

rfa_status rfa_set_wait_limit_ns(uint64_t ns) {
    const uint64_t v = ns == 0 ? rfa::kWaitLimitNs : ns;
    if (cudaDeviceSynchronize() != cudaSuccess) return RFA_ERR_CUDA;
    return cudaMemcpyToSymbol(rfa::g_wait_limit_ns, &v, sizeof v) == cudaSuccess ? RFA_OK : RFA_ERR_CUDA;
}

rfa_status rfa_set_hold_items(int32_t on) {
    const int32_t v = on != 0 ? 1 : 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return RFA_ERR_CUDA;
    return cudaMemcpyToSymbol(rfa::g_hold_items, &v, sizeof v) == cudaSuccess ? RFA_OK : RFA_ERR_CUDA;
}

rfa_status rfa_rope_sincos(const int32_t* positionIds, const float* invFreq, const int32_t* seqLens, int32_t batch,
                           int32_t ntokens, int32_t headSize, rfa_dtype outType, void* sinOut, void* cosOut,
                           void* stream) {
    if (!positionIds || !invFreq || !seqLens || !sinOut || !cosOut) return RFA_ERR_INVALID_ARG;
    if (outType == RFA_DT_UNDEFINED) return RFA_ERR_INVALID_ARG;
    if (outType != RFA_DT_FP16 && outType != RFA_DT_BF16 && outType != RFA_DT_FP32) return RFA_ERR_INVALID_ARG;
    if (batch < 1 || batch > rfa::kMaxSeqs) return RFA_ERR_INVALID_ARG;
    if (ntokens < 1 || ntokens > 256000) return RFA_ERR_INVALID_ARG;
    if (headSize < 32 || headSize > 2048 || headSize % 32 != 0) return RFA_ERR_INVALID_ARG;
    if (!aligned(invFreq, 16) || !aligned(sinOut, 16) || !aligned(cosOut, 16)) return RFA_ERR_INVALID_ARG;
    const int64_t work = static_cast<int64_t>(ntokens) * (headSize / 16);
    cudaStream_t st = as_stream(stream);
    const size_t esize = outType == RFA_DT_FP32 ? 4 : 2;
    const bool stream_out = streams(2.0 * static_cast<double>(ntokens) * headSize * esize);  // sin + cos
    switch (outType) {
        case RFA_DT_FP16:
            launch_sincos<__half>(stream_out, work, st, positionIds, invFreq, seqLens, batch, ntokens, headSize,
                                  sinOut, cosOut);
            break;
        case RFA_DT_BF16:
            launch_sincos<__nv_bfloat16>(stream_out, work, st, positionIds, invFreq, seqLens, batch, ntokens,
                                         headSize, sinOut, cosOut);
            break;
        default:
            launch_sincos<float>(stream_out, work, st, positionIds, invFreq, seqLens, batch, ntokens, headSize,
                                 sinOut, cosOut);
            break;
    }
    return cudaGetLastError() == cudaSuccess ? RFA_OK : RFA_ERR_CUDA;
}

}  // extern "C"

namespace {

template <bool kFP16, typename TabT>
void launch_rope_apply(const rfa::RopeApplyArgs& a, bool interleaved, bool stream_mem, uint32_t work,
                       cudaStream_t st) {
    auto kern = interleaved ? (stream_mem ? rfa::rope_apply_kernel<kFP16, TabT, true, true>
                                          : rfa::rope_apply_kernel<kFP16, TabT, true, false>)
                            : (stream_mem ? rfa::rope_apply_kernel<kFP16, TabT, false, true>
                                          : rfa::rope_apply_kernel<kFP16, TabT, false, false>);
    kern<<<resident_grid(kern, work, 256), 256, 0, st>>>(a);
}

}  // namespace

extern "C" {

rfa_status rfa_rope_apply(const rfa_rope_apply_params* p, const void* q, const void* k, const void* sin,
                          const void* cos, void* q_out, void* k_out, const int32_t* cache_slots, void* k_cache,
                          int64_t cache_rows, void* stream) {
    if (!p || !sin || !cos) return RFA_ERR_INVALID_ARG;
    if (p->layout != RFA_LAYOUT_BNSD && p->layout != RFA_LAYOUT_TND) return RFA_ERR_INVALID_ARG;
    const bool bnsd = p->layout == RFA_LAYOUT_BNSD;
    int64_t R;
    if (bnsd) {
        if (p->B < 1 || p->S < 1) return RFA_ERR_INVALID_ARG;
        R = static_cast<int64_t>(p->B) * p->S;
    } else {
        if (p->T < 1) return RFA_ERR_INVALID_ARG;
        R = p->T;
    }
    if (p->Hq < 0 || p->Hkv < 0 || p->Hq + p->Hkv < 1) return RFA_ERR_INVALID_ARG;
    if (p->D < 16 || p->D > 512 || p->D % 16 != 0) return RFA_ERR_INVALID_ARG;
    if (p->interleaved != 0 && p->interleaved != 1) return RFA_ERR_INVALID_ARG;
    if (p->io_dtype != RFA_DT_BF16 && p->io_dtype != RFA_DT_FP16)
        return p->io_dtype == RFA_DT_FP32 ? RFA_ERR_UNSUPPORTED : RFA_ERR_INVALID_ARG;
    if (p->table_dtype != RFA_DT_BF16 && p->table_dtype != RFA_DT_FP16 && p->table_dtype != RFA_DT_FP32)
        return RFA_ERR_INVALID_ARG;
    // q: given exactly when it has heads, with somewhere to write; k likewise (k_out and/or the cache)
    if ((q != nullptr) != (p->Hq > 0) || (p->Hq > 0 && !q_out)) return RFA_ERR_INVALID_ARG;
    if ((k != nullptr) != (p->Hkv > 0)) return RFA_ERR_INVALID_ARG;
    if ((cache_slots != nullptr) != (k_cache != nullptr)) return RFA_ERR_INVALID_ARG;
    if (k_cache && (p->Hkv < 1 || cache_rows < 1)) return RFA_ERR_INVALID_ARG;
    if (p->Hkv > 0 && !k_out && !k_cache) return RFA_ERR_INVALID_ARG;
    for (const void* ptr : {static_cast<const void*>(q), k, sin, cos, static_cast<const void*>(q_out),
                            static_cast<const void*>(k_out), static_cast<const void*>(k_cache)})
        if (ptr && !aligned(ptr, 16)) return RFA_ERR_INVALID_ARG;
    if (cache_slots && !aligned(cache_slots, 4)) return RFA_ERR_INVALID_ARG;
    const int64_t hgroups = (p->Hq + p->Hkv + rfa::kApplyHeads - 1) / rfa::kApplyHeads;
    const int64_t work = R * hgroups * (p->D / 16);
    if (work >= (int64_t{1} << 31)) return RFA_ERR_UNSUPPORTED;
    rfa::RopeApplyArgs a;
    a.q = q;
    a.k = k;
    a.sin_t = sin;
    a.cos_t = cos;
    a.q_out = q_out;
    a.k_out = k_out;
    a.slots = cache_slots;
    a.cache = k_cache;
    a.cache_rows = cache_rows;
    a.bnsd = bnsd ? 1 : 0;
    a.R = static_cast<int32_t>(R);
    a.S = bnsd ? p->S : 1;
    a.Hq = p->Hq;
    a.Hkv = p->Hkv;
    a.D = p->D;
    const bool fp16 = p->io_dtype == RFA_DT_FP16;
    const bool inter = p->interleaved != 0;
    // q and k rows read, rotated rows written (k twice when it also goes to the cache)
    const double row_bytes = static_cast<double>(p->D) * 2.0;
    const bool sm = streams(static_cast<double>(R) * row_bytes *
                            (2.0 * p->Hq + (1.0 + (k_out ? 1.0 : 0.0) + (k_cache ? 1.0 : 0.0)) * p->Hkv));
    const uint32_t w = static_cast<uint32_t>(work);
    cudaStream_t st = as_stream(stream);
    switch (p->table_dtype) {
        case RFA_DT_FP16:
            fp16 ? launch_rope_apply<true, __half>(a, inter, sm, w, st) : launch_rope_apply<false, __half>(a, inter, sm, w, st);
            break;
        case RFA_DT_BF16:
            fp16 ? launch_rope_apply<true, __nv_bfloat16>(a, inter, sm, w, st)
                 : launch_rope_apply<false, __nv_bfloat16>(a, inter, sm, w, st);
            break;
        default:
            fp16 ? launch_rope_apply<true, float>(a, inter, sm, w, st) : launch_rope_apply<false, float>(a, inter, sm, w, st);
            break;
    }
    return cudaGetLastError() == cudaSuccess ? RFA_OK : RFA_ERR_CUDA;
}

}  // extern "C"

namespace {

template <bool kFP16, typename TabT>
void launch_kv_cache(const rfa::KvCacheArgs& a, bool interleaved, bool stream_mem, uint32_t work, cudaStream_t st) {
    auto kern = interleaved ? (stream_mem ? rfa::kv_norm_rope_cache_kernel<kFP16, TabT, true, true>
                                          : rfa::kv_norm_rope_cache_kernel<kFP16, TabT, true, false>)
                            : (stream_mem ? rfa::kv_norm_rope_cache_kernel<kFP16, TabT, false, true>
                                          : rfa::kv_norm_rope_cache_kernel<kFP16, TabT, false, false>);
    kern<<<resident_grid(kern, work, 256), 256, 0, st>>>(a);
}

}  // namespace

extern "C" {

rfa_status rfa_kv_rms_norm_rope_cache(const rfa_kv_cache_params* p, const void* k, const void* v, const float* gamma,
                                      const void* sin, const void* cos, const int32_t* slots, void* k_cache,
                                      void* v_cache, int64_t cache_rows, void* stream) {
    if (!p || !k || !v || !gamma || !sin || !cos || !slots || !k_cache || !v_cache) return RFA_ERR_INVALID_ARG;
    if (p->T < 1 || p->Hkv < 1 || cache_rows < 1) return RFA_ERR_INVALID_ARG;
    if (p->D < 16 || p->D > 512 || (p->D & (p->D - 1)) != 0) return RFA_ERR_INVALID_ARG;
    if (p->interleaved != 0 && p->interleaved != 1) return RFA_ERR_INVALID_ARG;
    if (!(p->eps >= 0.0f) || !std::isfinite(p->eps)) return RFA_ERR_INVALID_ARG;
    if (p->io_dtype != RFA_DT_BF16 && p->io_dtype != RFA_DT_FP16)
        return p->io_dtype == RFA_DT_FP32 ? RFA_ERR_UNSUPPORTED : RFA_ERR_INVALID_ARG;
    if (p->table_dtype != RFA_DT_BF16 && p->table_dtype != RFA_DT_FP16 && p->table_dtype != RFA_DT_FP32)
        return RFA_ERR_INVALID_ARG;
    for (const void* ptr : {k, v, static_cast<const void*>(gamma), sin, cos, static_cast<const void*>(k_cache),
                            static_cast<const void*>(v_cache)})
        if (!aligned(ptr, 16)) return RFA_ERR_INVALID_ARG;
    if (!aligned(slots, 4)) return RFA_ERR_INVALID_ARG;
    const int64_t work = static_cast<int64_t>(p->T) * p->Hkv * (p->D / 16);
    if (work >= (int64_t{1} << 31)) return RFA_ERR_UNSUPPORTED;
    rfa::KvCacheArgs a;
    a.k = k;
    a.v = v;
    a.gamma = gamma;
    a.sin_t = sin;
    a.cos_t = cos;
    a.slots = slots;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.cache_rows = cache_rows;
    a.T = p->T;
    a.Hkv = p->Hkv;
    a.D = p->D;
    a.eps = p->eps;
    const bool fp16 = p->io_dtype == RFA_DT_FP16, inter = p->interleaved != 0;
    // k and v rows read, both caches written
    const bool sm = streams(4.0 * static_cast<double>(p->T) * p->Hkv * p->D * 2.0);
    const uint32_t w = static_cast<uint32_t>(work);
    cudaStream_t st = as_stream(stream);
    switch (p->table_dtype) {
        case RFA_DT_FP16:
            fp16 ? launch_kv_cache<true, __half>(a, inter, sm, w, st) : launch_kv_cache<false, __half>(a, inter, sm, w, st);
            break;
        case RFA_DT_BF16:
            fp16 ? launch_kv_cache<true, __nv_bfloat16>(a, inter, sm, w, st)
                 : launch_kv_cache<false, __nv_bfloat16>(a, inter, sm, w, st);
            break;
        default:
            fp16 ? launch_kv_cache<true, float>(a, inter, sm, w, st) : launch_kv_cache<false, float>(a, inter, sm, w, st);
            break;
    }
    return cudaGetLastError() == cudaSuccess ? RFA_OK : RFA_ERR_CUDA;
}

size_t rfa_fused_rope_attention_workspace(const rfa_attn_params* p, int64_t ntokens) {
    if (validate_attn(p) != RFA_OK || ntokens < 1) return 0;
    return workspace_bytes(ntokens, p->D, p->B);
}

}  // extern "C"

namespace {

rfa_status check_common(const rfa_attn_params* p, const int32_t* seqLens_host, int64_t* T_out) {
    rfa_status vs = validate_attn(p);
    if (vs != RFA_OK) return vs;
    if (p->layout == RFA_LAYOUT_TND) {
        if (!seqLens_host) return RFA_ERR_INVALID_ARG;
        for (int b = 0; b < p->B; ++b)
            if (seqLens_host[b] <= 0) return RFA_ERR_INVALID_ARG;
    }
    const int64_t T = total_tokens(p, seqLens_host);
    if (T < 1 || T > (int64_t{1} << 31) / 4 - 1) return RFA_ERR_INVALID_ARG;
    *T_out = T;
    return RFA_OK;
}

rfa_status enqueue_table(const rfa_attn_params* p, int64_t T, const int32_t* position, const int32_t* seqLens_host,
                         const float* invFreq, void* workspace, cudaStream_t st) {
    const bool tnd = p->layout == RFA_LAYOUT_TND;
    const int D = p->D;
    const int half = D / 2;
    rfa::TableArgs ta;
    std::memset(&ta, 0, sizeof ta);
    ta.pos = position;
    ta.inv_dev = invFreq;
    ta.table = static_cast<uint32_t*>(workspace);
    ta.seeds = reinterpret_cast<rfa::RopeSeed*>(static_cast<char*>(workspace) + table_bytes(T, D));
    ta.sched = sched_of(workspace, T, D, p->B);
    ta.ntokens = static_cast<int32_t>(T);
    ta.npos = static_cast<int32_t>(T);
    ta.inv_dev_rows = p->B;
    ta.half = half;
    ta.nseg = p->B;
    ta.uniform_len = tnd ? 0 : p->S;
    if (tnd) {
        int64_t acc = 0;
        for (int b = 0; b < p->B; ++b) {
            ta.cum[b] = static_cast<int32_t>(acc);
            acc += seqLens_host[b];
        }
        ta.cum[p->B] = static_cast<int32_t>(acc);
    }
    if (!invFreq) {
        if (!tnd || !p->ntk_enable) {
            ta.inv_host_rows = 1;
            inv_freq_row(ntk_base(p, tnd ? 0 : p->S), D, ta.inv_host);
        } else {
            ta.inv_host_rows = p->B;
            for (int b = 0; b < p->B; ++b) inv_freq_row(ntk_base(p, seqLens_host[b]), D, ta.inv_host + b * half);
        }
    }
    // seeds first: the table kernel clears the consecutive flag the seed kernel sets
    rfa::rope_seed_kernel<<<p->B, 64, 0, st>>>(ta);
    if (cudaGetLastError() != cudaSuccess) return RFA_ERR_CUDA;
    rfa::rope_table_kernel<<<grid_for(T * (half / 8), 256), 256, 0, st>>>(ta);
    return cudaGetLastError() == cudaSuccess ? RFA_OK : RFA_ERR_CUDA;
}

rfa_status enqueue_attention(const rfa_attn_params* p, int64_t T, const void* q, const void* k, const void* v,
                             const int32_t* seqLens_host, void* out, void* table, cudaStream_t st) {
    const bool tnd = p->layout == RFA_LAYOUT_TND;
    const int D = p->D;
    rfa::AttnArgs aa;
    std::memset(&aa, 0, sizeof aa);
    aa.out = out;
    aa.seeds = reinterpret_cast<const rfa::RopeSeed*>(static_cast<const char*>(table) + table_bytes(T, D));
    aa.table = static_cast<const uint32_t*>(table);
    aa.sched = sched_of(table, T, D, p->B);
    aa.out_elems = T * p->Hq * D;
    aa.ntok = static_cast<int32_t>(T);
    aa.layout = tnd ? 1 : 0;
    aa.B = p->B;
    aa.Hq = p->Hq;
    aa.Hkv = p->Hkv;
    aa.G = p->Hq / p->Hkv;
    aa.S = tnd ? 0 : p->S;
    aa.causal = p->causal ? 1 : 0;
    // two query tiles per CTA: two heads of one kv group when G is even, else consecutive tiles of one head
    const bool pair_heads = (aa.G % 2) == 0;
    aa.pair_heads = pair_heads ? 1 : 0;
    const float scale = p->scale > 0.0f ? p->scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
    aa.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    const bool fp16 = p->io_dtype == RFA_DT_FP16;
    const uint64_t esz = 2;
    CUtensorMap mq, mk, mv;
    bool ok;
    if (!tnd) {
        const int64_t nqt = (p->S + rfa::kBlockM - 1) / rfa::kBlockM;
        const int64_t items = static_cast<int64_t>(rfa::items_per_sequence(p->Hq, static_cast<int32_t>(nqt), pair_heads)) * p->B;
        if (items > 0x7fffffff) return RFA_ERR_UNSUPPORTED;
        aa.n_items = static_cast<int32_t>(items);
        ok = make_map(&mq, q, fp16, D, p->S, static_cast<uint64_t>(p->B) * p->Hq, D * esz, p->S * D * esz, 64,
                      rfa::kBlockM, 1) &&
             make_map(&mk, k, fp16, D, p->S, static_cast<uint64_t>(p->B) * p->Hkv, D * esz, p->S * D * esz, 64,
                      rfa::kBlockN, 1) &&
             make_map(&mv, v, fp16, D, p->S, static_cast<uint64_t>(p->B) * p->Hkv, D * esz, p->S * D * esz, 64,
                      rfa::kBlockN, 1);
    } else {
        // sequences sorted by query-tile count, descending (longest first)
        int order[rfa::kMaxSeqs];
        int starts[rfa::kMaxSeqs];
        int64_t acc = 0;
        for (int b = 0; b < p->B; ++b) {
            order[b] = b;
            starts[b] = static_cast<int>(acc);
            acc += seqLens_host[b];
        }
        std::stable_sort(order, order + p->B, [&](int x, int y) { return seqLens_host[x] > seqLens_host[y]; });
        aa.nseg = p->B;
        int64_t items = 0;
        for (int i = 0; i < p->B; ++i) {
            const int b = order[i];
            aa.seg_start[i] = starts[b];
            aa.seg_orig[i] = b;
            aa.seg_len[i] = seqLens_host[b];
            aa.seg_tiles[i] = (seqLens_host[b] + rfa::kBlockM - 1) / rfa::kBlockM;
            aa.seg_item0[i] = static_cast<int32_t>(std::min<int64_t>(items, 0x7fffffff));
            items += rfa::items_per_sequence(p->Hq, aa.seg_tiles[i], pair_heads);
        }
        aa.seg_item0[p->B] = static_cast<int32_t>(std::min<int64_t>(items, 0x7fffffff));
        if (items > 0x7fffffff) return RFA_ERR_UNSUPPORTED;
        aa.n_items = static_cast<int32_t>(items);
        ok = make_map(&mq, q, fp16, D, p->Hq, T, D * esz, static_cast<uint64_t>(p->Hq) * D * esz, 64, 1,
                      rfa::kBlockM) &&
             make_map(&mk, k, fp16, D, p->Hkv, T, D * esz, static_cast<uint64_t>(p->Hkv) * D * esz, 64, 1,
                      rfa::kBlockN) &&
             make_map(&mv, v, fp16, D, p->Hkv, T, D * esz, static_cast<uint64_t>(p->Hkv) * D * esz, 64, 1,
                      rfa::kBlockN);
    }
    CUtensorMap mt;
    ok = ok && make_table_map(&mt, table, static_cast<uint64_t>(T), D);
    if (!ok) return RFA_ERR_CUDA;
    // the output as the query's geometry, for the kernel's tiled stores of whole output tiles;
    // when it cannot be described (e.g. not 16-byte aligned) the kernel stores rows itself
    CUtensorMap mo = mq;
    aa.tma_out = (tnd ? make_map(&mo, out, fp16, D, p->Hq, T, D * esz, static_cast<uint64_t>(p->Hq) * D * esz, 64,
                                 1, rfa::kBlockM)
                      : make_map(&mo, out, fp16, D, p->S, static_cast<uint64_t>(p->B) * p->Hq, D * esz,
                                 p->S * D * esz, 64, rfa::kBlockM, 1))
                     ? 1
                     : 0;
    if (!aa.tma_out) mo = mq;
    const bool adj = p->rope_interleaved != 0;
    if (D == 128) {
        if (adj)
            return fp16 ? launch_attn<128, true, true>(mq, mk, mv, mt, mo, aa, st)
                        : launch_attn<128, false, true>(mq, mk, mv, mt, mo, aa, st);
        return fp16 ? launch_attn<128, true, false>(mq, mk, mv, mt, mo, aa, st)
                    : launch_attn<128, false, false>(mq, mk, mv, mt, mo, aa, st);
    }
    if (adj)
        return fp16 ? launch_attn<64, true, true>(mq, mk, mv, mt, mo, aa, st)
                    : launch_attn<64, false, true>(mq, mk, mv, mt, mo, aa, st);
    return fp16 ? launch_attn<64, true, false>(mq, mk, mv, mt, mo, aa, st)
                : launch_attn<64, false, false>(mq, mk, mv, mt, mo, aa, st);
}

}  // namespace

extern "C" {

rfa_status rfa_rope_attention_table(const rfa_attn_params* p, const int32_t* position, const int32_t* seqLens_host,
                                    const float* invFreq, void* workspace, size_t ws_bytes, void* stream) {
    int64_t T = 0;
    rfa_status vs = check_common(p, seqLens_host, &T);
    if (vs != RFA_OK) return vs;
    if (!position) return RFA_ERR_INVALID_ARG;
    if (invFreq && !aligned(invFreq, 16)) return RFA_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < workspace_bytes(T, p->D, p->B) || !aligned(workspace, 256)) return RFA_ERR_WORKSPACE;
    return enqueue_table(p, T, position, seqLens_host, invFreq, workspace, as_stream(stream));
}

rfa_status rfa_fused_rope_attention_with_table(const rfa_attn_params* p, const void* q, const void* k, const void* v,
                                               const int32_t* seqLens_host, void* out, void* workspace,
                                               size_t ws_bytes, void* stream) {
    int64_t T = 0;
    rfa_status vs = check_common(p, seqLens_host, &T);
    if (vs != RFA_OK) return vs;
    if (!q || !k || !v || !out) return RFA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return RFA_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < workspace_bytes(T, p->D, p->B) || !aligned(workspace, 256)) return RFA_ERR_WORKSPACE;
    return enqueue_attention(p, T, q, k, v, seqLens_host, out, workspace, as_stream(stream));
}

rfa_status rfa_fused_rope_attention(const rfa_attn_params* p, const void* q, const void* k, const void* v,
                                    const int32_t* position, const int32_t* seqLens_host, const float* invFreq,
                                    void* out, void* workspace, size_t ws_bytes, void* stream) {
    int64_t T = 0;
    rfa_status vs = check_common(p, seqLens_host, &T);
    if (vs != RFA_OK) return vs;
    if (!q || !k || !v || !position || !out) return RFA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return RFA_ERR_INVALID_ARG;
    if (invFreq && !aligned(invFreq, 16)) return RFA_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < workspace_bytes(T, p->D, p->B) || !aligned(workspace, 256)) return RFA_ERR_WORKSPACE;
    cudaStream_t st = as_stream(stream);
    rfa_status r = enqueue_table(p, T, position, seqLens_host, invFreq, workspace, st);
    if (r != RFA_OK) return r;
    return enqueue_attention(p, T, q, k, v, seqLens_host, out, workspace, st);
}

}  // extern "C"

// ---------------------------------------------------------------- workspace-free variant
// Some callers cannot allocate device memory on the path that calls us: code
// running while a stream is being captured into a CUDA graph, plugins whose
// host framework owns every device buffer and only hands a kernel its inputs
// and outputs, and real-time callers that may not block on an allocator.
// rfa_fused_rope_attention_noalloc serves them with a fixed scratch area that
// lives in this library's module for as long as the library is loaded.
namespace {

constexpr int64_t kNoAllocMaxTokens = 65536;  // T limit of the fixed scratch
constexpr int kNoAllocMaxSeqs = 16;           // sequences (BNSD: batches) limit
constexpr size_t kNoAllocTableBytes = static_cast<size_t>(kNoAllocMaxTokens) * 128 * 2;  // D <= 128
constexpr size_t kNoAllocSeedBytes = (kNoAllocMaxSeqs * sizeof(rfa::RopeSeed) + 255) / 256 * 256;
constexpr size_t kNoAllocBytes = kNoAllocTableBytes + kNoAllocSeedBytes + kSchedBytes;

}  // namespace

// The scratch itself: one copy per device that loads the module (~16.8 MB).
// Host code must not pass this symbol to a kernel (on the host it is only a
// stand-in); its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

namespace {

// Device address of g_noalloc_scratch on the current device, looked up once per
// device (the first call on a device does it; make that call before any
// stream capture begins).
rfa_status noalloc_scratch(void** out) {
    static std::mutex mu;
    static void* ptrs[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RFA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(mu);
    if (!ptrs[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return RFA_ERR_CUDA;
        ptrs[dev] = p;
    }
    *out = ptrs[dev];
    return RFA_OK;
}

}  // namespace

extern "C" {

rfa_status rfa_fused_rope_attention_noalloc(const rfa_attn_params* p, const void* q, const void* k, const void* v,
                                            const int32_t* position, const int32_t* seqLens_host,
                                            const float* invFreq, void* out, void* stream) {
    int64_t T = 0;
    rfa_status vs = check_common(p, seqLens_host, &T);
    if (vs != RFA_OK) return vs;
    if (!q || !k || !v || !position || !out) return RFA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return RFA_ERR_INVALID_ARG;
    if (invFreq && !aligned(invFreq, 16)) return RFA_ERR_INVALID_ARG;
    // The fixed scratch bounds the problem: reject what does not fit.
    if (T > kNoAllocMaxTokens || p->B > kNoAllocMaxSeqs || workspace_bytes(T, p->D, p->B) > kNoAllocBytes)
        return RFA_ERR_WORKSPACE;
    void* scratch = nullptr;
    rfa_status r = noalloc_scratch(&scratch);
    if (r != RFA_OK) return r;
    // Nothing in the scratch needs to start at zero: the table and seed
    // kernels write every byte the attention kernel reads, and zero its work
    // counters.
    cudaStream_t st = as_stream(stream);
    r = enqueue_table(p, T, position, seqLens_host, invFreq, scratch, st);
    if (r != RFA_OK) return r;
    return enqueue_attention(p, T, q, k, v, seqLens_host, out, scratch, st);
}

}  // extern "C"

// ---------------------------------------------------------------- decode over a KV cache
namespace {

struct DecodePlan {
    int32_t splits, chunk;
    int64_t rq;  // query rows B * Hq * Sq
    size_t po_bytes, pml_bytes, total;
};

rfa_status decode_validate(const rfa_decode_params* p) {
    if (!p) return RFA_ERR_INVALID_ARG;
    if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->Sq < 1 || p->Smax < 1) return RFA_ERR_INVALID_ARG;
    if (p->Hq % p->Hkv != 0) return RFA_ERR_INVALID_ARG;
    if (p->max_kv_len < p->Sq || p->max_kv_len > p->Smax) return RFA_ERR_INVALID_ARG;
    if (p->io_dtype != RFA_DT_BF16 && p->io_dtype != RFA_DT_FP16)
        return p->io_dtype == RFA_DT_UNDEFINED ? RFA_ERR_INVALID_ARG : RFA_ERR_UNSUPPORTED;
    if (p->rope_interleaved != 0 && p->rope_interleaved != 1) return RFA_ERR_INVALID_ARG;
    if (!(p->scale >= 0.0f) || !std::isfinite(p->scale)) return RFA_ERR_INVALID_ARG;
    if (!(p->rope_base > 0.0) || !std::isfinite(p->rope_base)) return RFA_ERR_INVALID_ARG;
    if (p->num_splits < 0) return RFA_ERR_INVALID_ARG;
    if ((p->D & 1) != 0 || p->D < 1) return RFA_ERR_INVALID_ARG;
    if (p->D != 64 && p->D != 128) return RFA_ERR_UNSUPPORTED;
    if ((p->Hq / p->Hkv) * p->Sq > rfa::kBlockM) return RFA_ERR_UNSUPPORTED;  // one query tile per kv group
    if (static_cast<int64_t>(p->B) * p->Smax >= (int64_t{1} << 31)) return RFA_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(p->B) * p->Hq * p->Sq >= (int64_t{1} << 31) / 256) return RFA_ERR_UNSUPPORTED;
    return RFA_OK;
}

// Keys of a sequence are split into whole key tiles across CTAs; one CTA is
// resident per SM, so B * Hkv * splits CTAs run in ceil(that / SMs) waves of
// about tiles / splits key tiles each.  The plan takes the split count with the
// least waves x (tiles per split + kSplitCost), kSplitCost being the fixed cost
// of a CTA (setup, query load and rotation, pipeline fill and drain, merge and
// store) in key tiles; ties go to fewer splits.  kSplitCost = 6 fits timings of
// 1 to 64 sequences over 4K-32K cached keys (32 query / 8 kv heads, D 128):
// e.g. 8 sequences x 32K keys run fastest as 2 splits, one wave of 128 CTAs
// that already saturates HBM.
constexpr int64_t kSplitCost = 6;
DecodePlan decode_plan(const rfa_decode_params* p) {
    DecodePlan pl;
    pl.rq = static_cast<int64_t>(p->B) * p->Hq * p->Sq;
    const int64_t groups = static_cast<int64_t>(p->B) * p->Hkv;
    const int32_t tiles = (p->max_kv_len + rfa::kBlockN - 1) / rfa::kBlockN;
    const int64_t sms = device_sms();
    int32_t per = tiles;
    if (p->num_splits > 0) {
        per = (tiles + std::min(p->num_splits, tiles) - 1) / std::min(p->num_splits, tiles);
    } else {
        // beyond about 8 waves more splits only add CTA costs
        const int64_t s_max = std::min<int64_t>(tiles, std::max<int64_t>(1, (8 * sms + groups - 1) / groups));
        int64_t best = -1;
        for (int32_t s = 1; s <= s_max; ++s) {
            const int32_t ps = (tiles + s - 1) / s;
            if (s > 1 && ps == (tiles + s - 2) / (s - 1)) continue;  // same split as s - 1
            const int64_t n = (tiles + ps - 1) / ps;
            const int64_t cost = ((groups * n + sms - 1) / sms) * (ps + kSplitCost);
            if (best < 0 || cost < best) {
                best = cost;
                per = ps;
            }
        }
    }
    pl.chunk = per * rfa::kBlockN;
    pl.splits = (p->max_kv_len + pl.chunk - 1) / pl.chunk;
    pl.po_bytes = pl.splits > 1 ? round_up(static_cast<size_t>(pl.splits) * pl.rq * p->D * 4, 256) : 0;
    pl.pml_bytes = pl.splits > 1 ? round_up(static_cast<size_t>(pl.splits) * pl.rq * 2 * 4, 256) : 0;
    pl.total = std::max<size_t>(256, pl.po_bytes + pl.pml_bytes);  // never 0: 0 reports invalid parameters
    return pl;
}

}  // namespace

extern "C" {

size_t rfa_decode_rope_attention_workspace(const rfa_decode_params* p) {
    if (decode_validate(p) != RFA_OK) return 0;
    return decode_plan(p).total;
}

rfa_status rfa_decode_rope_attention(const rfa_decode_params* p, const void* q, const void* k_cache,
                                     const void* v_cache, const int32_t* q_pos, const int32_t* kv_lens,
                                     const float* invFreq, void* out, void* workspace, size_t ws_bytes,
                                     void* stream) {
    rfa_status vs = decode_validate(p);
    if (vs != RFA_OK) return vs;
    if (!q || !k_cache || !v_cache || !q_pos || !kv_lens || !out) return RFA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16))
        return RFA_ERR_INVALID_ARG;
    if (invFreq && !aligned(invFreq, 16)) return RFA_ERR_INVALID_ARG;
    const DecodePlan pl = decode_plan(p);
    if (!workspace || ws_bytes < pl.total || !aligned(workspace, 256)) return RFA_ERR_WORKSPACE;
    const int D = p->D;
    const bool fp16 = p->io_dtype == RFA_DT_FP16;
    cudaStream_t st = as_stream(stream);
    char* ws = static_cast<char*>(workspace);
    rfa::AttnArgs aa;
    std::memset(&aa, 0, sizeof aa);
    // the query rows' cos/sin are formed in the kernel from their positions and frequencies
    aa.dec_qpos = q_pos;
    aa.dec_inv = invFreq;
    if (!invFreq) inv_freq_row(p->rope_base, D, aa.dec_inv_host);
    aa.out = out;
    aa.seeds = nullptr;
    aa.layout = 1;  // cache rows token-major: [B * Smax, Hkv, D]
    aa.B = p->B;
    aa.Hq = p->Hq;
    aa.Hkv = p->Hkv;
    aa.G = p->Hq / p->Hkv;
    aa.causal = p->causal ? 1 : 0;
    const float scale = p->scale > 0.0f ? p->scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
    aa.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    aa.n_items = p->B * p->Hkv * pl.splits;
    aa.dec_Sq = p->Sq;
    aa.dec_Smax = p->Smax;
    aa.dec_splits = pl.splits;
    aa.dec_chunk = pl.chunk;
    aa.dec_max_len = p->max_kv_len;
    aa.kv_lens = kv_lens;
    aa.out_elems = pl.rq * D;
    aa.ntok = p->B * p->Smax;
    aa.part_o = pl.splits > 1 ? reinterpret_cast<float*>(ws) : nullptr;
    aa.part_ml = pl.splits > 1 ? reinterpret_cast<float*>(ws + pl.po_bytes) : nullptr;
    const uint64_t esz = 2, rows_cache = static_cast<uint64_t>(p->B) * p->Smax;
    CUtensorMap mq, mk, mv;
    bool ok = make_map(&mq, q, fp16, D, 1, static_cast<uint64_t>(pl.rq), D * esz, D * esz, 64, 1, rfa::kBlockM) &&
              make_map(&mk, k_cache, fp16, D, p->Hkv, rows_cache, D * esz, static_cast<uint64_t>(p->Hkv) * D * esz, 64,
                       1, rfa::kBlockN) &&
              make_map(&mv, v_cache, fp16, D, p->Hkv, rows_cache, D * esz, static_cast<uint64_t>(p->Hkv) * D * esz, 64,
                       1, rfa::kBlockN);
    if (!ok) return RFA_ERR_CUDA;
    const bool adj = p->rope_interleaved != 0;
    rfa_status r;
    const CUtensorMap& mo = mq;  // decode stores its rows itself
    const CUtensorMap& mt = mq;  // and reads no table (the kernel forms the query rows' cos/sin)
    if (D == 128) {
        if (adj)
            r = fp16 ? launch_attn<128, true, true, true>(mq, mk, mv, mt, mo, aa, st)
                     : launch_attn<128, false, true, true>(mq, mk, mv, mt, mo, aa, st);
        else
            r = fp16 ? launch_attn<128, true, false, true>(mq, mk, mv, mt, mo, aa, st)
                     : launch_attn<128, false, false, true>(mq, mk, mv, mt, mo, aa, st);
    } else {
        if (adj)
            r = fp16 ? launch_attn<64, true, true, true>(mq, mk, mv, mt, mo, aa, st)
                     : launch_attn<64, false, true, true>(mq, mk, mv, mt, mo, aa, st);
        else
            r = fp16 ? launch_attn<64, true, false, true>(mq, mk, mv, mt, mo, aa, st)
                     : launch_attn<64, false, false, true>(mq, mk, mv, mt, mo, aa, st);
    }
    if (r != RFA_OK || pl.splits == 1) return r;
    // the combine kernel as a programmatic dependent launch: its blocks are placed while the
    // decode grid finishes and wait (griddepcontrol.wait) for its partials
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(grid_for(pl.rq * (D / 8), 256)));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float* po = aa.part_o;
    const float* pml = aa.part_ml;
    const int32_t rows = static_cast<int32_t>(pl.rq), Dc = D, splits = pl.splits;
    const cudaError_t e = fp16 ? cudaLaunchKernelEx(&cfg, rfa::decode_combine_kernel<true>, po, pml, out, rows, Dc, splits)
                               : cudaLaunchKernelEx(&cfg, rfa::decode_combine_kernel<false>, po, pml, out, rows, Dc, splits);
    return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? RFA_OK : RFA_ERR_CUDA;
}

}  // extern "C"
