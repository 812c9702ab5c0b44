// stream_mem.cuh -- 16-byte global loads and stores with an optional
// evict-first cache hint (ld.global.cs / st.global.cs).  The elementwise
// kernels (sin/cos table, Rope operator, RMSNorm + RoPE + cache) read and
// write each byte once; when a launch moves more than half of L2, nothing it
// touches can stay resident for a later reader, and marking its lines
// evict-first keeps them from displacing the lines still in use.  The host
// chooses per launch.  Both forms are ordinary coherent accesses, so an output
// may alias an input.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

namespace rfa {

template <bool kStream>
__device__ __forceinline__ uint4 ldg128(const void* p) {
    if constexpr (kStream) {
        uint4 v;
        asm volatile("ld.global.cs.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "l"(p)
                     : "memory");
        return v;
    } else {
        return *reinterpret_cast<const uint4*>(p);
    }
}

template <bool kStream>
__device__ __forceinline__ void stg128(void* p, uint4 v) {
    if constexpr (kStream)
        asm volatile("st.global.cs.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                     : "memory");
    else
        *reinterpret_cast<uint4*>(p) = v;
}

}  // namespace rfa
