// common.cuh — device helpers shared by the KDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define KDA_DEVICE __device__ __forceinline__

namespace kda {

// ---------------------------------------------------------------- scalar I/O
template <typename T> KDA_DEVICE float to_f32(T x);
template <> KDA_DEVICE float to_f32<float>(float x) { return x; }
template <> KDA_DEVICE float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> KDA_DEVICE T from_f32(float x);
template <> KDA_DEVICE float from_f32<float>(float x) { return x; }
template <> KDA_DEVICE __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

template <typename T> KDA_DEVICE float ld_f32(const T *p) { return to_f32<T>(*p); }

// Load 4 consecutive elements (8 bytes for bf16, 16 bytes for fp32) as floats.
// The address must be aligned to 4 elements.
KDA_DEVICE void ld4(const float *p, float (&o)[4])
{
    const float4 t = *reinterpret_cast<const float4 *>(p);
    o[0] = t.x; o[1] = t.y; o[2] = t.z; o[3] = t.w;
}
KDA_DEVICE void ld4(const __nv_bfloat16 *p, float (&o)[4])
{
    const uint2 t = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&t.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&t.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    o[0] = fa.x; o[1] = fa.y; o[2] = fb.x; o[3] = fb.y;
}
KDA_DEVICE void st4(float *p, const float (&v)[4])
{
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
KDA_DEVICE void st4(__nv_bfloat16 *p, const float (&v)[4])
{
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 t;
    t.x = *reinterpret_cast<uint32_t *>(&a);
    t.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = t;
}

// ---------------------------------------------------------------- math
KDA_DEVICE float sigmoidf_(float x) { return 1.0f / (1.0f + __expf(-x)); }
KDA_DEVICE float siluf_(float x) { return x / (1.0f + __expf(-x)); }
// log(1 + e^x) without overflow
KDA_DEVICE float softplusf_(float x) { return x > 0.0f ? x + log1pf(__expf(-x)) : log1pf(__expf(x)); }

// The tokens of sequence b: rows row0 .. row0 + len - 1 of the flattened [tokens, H, d]
// tensors.  Fixed length (cu == nullptr): row0 = b T, len = T.  Packed variable length:
// row0 = cu[b], len = cu[b + 1] - cu[b], both clamped into [0, T] (T = total tokens), so
// that no access leaves the buffers whatever the offsets hold.
struct SeqSpan {
    int row0, len;
};
KDA_DEVICE SeqSpan seq_span(const int *cu, int b, int T)
{
    if (!cu) return SeqSpan{b * T, T};
    const int s = min(max(cu[b], 0), T);
    const int e = min(max(cu[b + 1], s), T);
    return SeqSpan{s, e - s};
}

KDA_DEVICE float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Device error word codes (written by a kernel whose bounded wait gave up).
enum : int { ERR_NONE = 0, ERR_MBAR_TIMEOUT = 1, ERR_BAD_LAUNCH = 2 };

KDA_DEVICE void raise_error(int *err, int code)
{
    if (err) atomicCAS(err, 0, code);
}

}  // namespace kda
