// gq_device.cuh -- device helpers shared by the libgq kernels: element loads,
// the quantize arithmetic, register top-m selection and team barriers.
//
// Arithmetic contract (the definitions in include/gq.h): every floating-point
// step that decides an output bit is one correctly rounded binary32 operation,
// written with the explicit-rounding intrinsics (__fmul_rn, __fadd_rn,
// __fdiv_rn, __frcp_rn), so the compiler cannot contract or reassociate it.
// The one exception is the reciprocal quotient of the fused row kernel, on
// paired f32x2 instructions that the code generator may contract: its code
// is decided by a guard whose margin covers either form (see round8_fast).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace gq {

constexpr int kF32 = 0;
constexpr int kBF16 = 1;

constexpr uint32_t kStatusNonfinite = 0x1u;
constexpr uint32_t kStatusRange = 0x2u;

// 1.5 * 2^23.  For |y| < 2^22, y + kMagic lies in [2^23, 2^24) where the
// binary32 spacing is 1, so the rounded sum is round_half_even(y) + kMagic
// (kMagic is even, so ties go to the even integer), its bit pattern is
// 0x4B400000 + round_half_even(y), and (y + kMagic) - kMagic is exact and
// gives +0.0 for a zero code.
constexpr float kMagic = 12582912.0f;
constexpr int32_t kMagicBits = 0x4B400000;

// Quotient approximation guard.  With r = RN(1/s) and y = RN(w * r):
//   |y - w/s| <= |w/s| * (2^-23 + 2^-48) and |RN(w/s) - w/s| <= |w/s| * 2^-24,
// so |y - RN(w/s)| < |w/s| * 2^-22.4.  Clipping gives |w| <= c, and c/s is at
// most 1.5 * qmax + 1 < 256 (the worst case is a binary16 subnormal scale
// rounded down), so |y - RN(w/s)| < 2^-14.4 < 2^-13.  The rounded code can
// differ only if a half-integer lies between y and RN(w/s); then y is within
// 2^-13 of that half-integer, i.e. |y - rint(y)| > 0.5 - 2^-13, and the exact
// quotient is computed instead.
constexpr float kNearHalf = 0.5f - 0.0001220703125f;   // 0.5 - 2^-13

// Scales with a normal reciprocal (and normal s) take the reciprocal path.
constexpr float kFastScaleMin = 2.350988701644575e-38f;  // 2^-125
constexpr float kFastScaleMax = 4.253529586511731e+37f;  // 2^125

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b16) {
    return __uint_as_float(b16 << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float x) {
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t*>(&h);
}

// |x| as an ordered key: non-negative binary32 values order like their bits.
__device__ __forceinline__ uint32_t abs_key(float x) {
    return __float_as_uint(x) & 0x7FFFFFFFu;
}

// Running average of quantize-dequantize snapshots (one binary32 array per
// tensor): kind 0 none, 1 copy (the first snapshot), 2 mean
// a + (x - a) * t with t = RN(1 / (n + 1)), 3 EMA RN(t * a) + RN(c * x) with
// t = decay and c = RN(1 - decay).  x is the snapshot as the model holds it.
constexpr int kAvgNone = 0, kAvgCopy = 1, kAvgMean = 2, kAvgEma = 3;

struct AvgOp {
    float* a;     // this row's averages (null: no average)
    float t;
    float c;
    int kind;
};

__device__ __forceinline__ float avg_update(float a, float x, const AvgOp& A) {
    if (A.kind == kAvgCopy) return x;
    if (A.kind == kAvgMean) return __fadd_rn(a, __fmul_rn(__fsub_rn(x, a), A.t));
    return __fadd_rn(__fmul_rn(A.t, a), __fmul_rn(A.c, x));
}

// Per-group quantization constants.
struct Scale {
    float c;       // clip value
    float s;       // scale used to quantize and dequantize
    float rcp;     // RN(1/s) when fast
    float qmaxf;
    bool fast;     // reciprocal path allowed
    bool zero;     // s == 0: every code is 0
};

// Clip -> scale (export mode rounds through binary16).  Sets *range on a
// binary16 overflow, returns h (binary16 bits, export mode) in *h_bits.
__device__ __forceinline__ Scale make_scale(uint32_t ckey, int qmax, bool export_mode,
                                            uint16_t* h_bits, bool* range) {
    Scale S;
    S.c = __uint_as_float(ckey);
    S.qmaxf = (float)qmax;
    float s32 = __fdiv_rn(S.c, S.qmaxf);
    float s = s32;
    *range = false;
    *h_bits = 0;
    if (export_mode) {
        __half h = __float2half_rn(s32);
        uint16_t hb = *reinterpret_cast<uint16_t*>(&h);
        *h_bits = hb;
        *range = (hb & 0x7FFFu) == 0x7C00u;
        s = __half2float(h);
    }
    S.s = s;
    S.zero = !(s != 0.0f);
    S.fast = (s >= kFastScaleMin) && (s <= kFastScaleMax);
    S.rcp = S.fast ? __frcp_rn(s) : 0.0f;
    return S;
}

// One element: returns the clamped, offset code b = kMagic + q (as a float).
__device__ __forceinline__ float quantize_offset(float w, const Scale& S) {
    float wc = fminf(fmaxf(w, -S.c), S.c);
    float y = S.fast ? __fmul_rn(wc, S.rcp) : __fdiv_rn(wc, S.s);
    float yM = __fadd_rn(y, kMagic);
    if (S.fast) {
        float d = fabsf(__fsub_rn(y, __fsub_rn(yM, kMagic)));
        if (d > kNearHalf) {
            y = __fdiv_rn(wc, S.s);
            yM = __fadd_rn(y, kMagic);
        }
    }
    float b = fminf(fmaxf(yM, kMagic - S.qmaxf), kMagic + S.qmaxf);
    return S.zero ? kMagic : b;
}

__device__ __forceinline__ int offset_to_code(float b) {
    return __float_as_int(b) - kMagicBits;
}

__device__ __forceinline__ float offset_to_dq(float b, const Scale& S) {
    return __fmul_rn(__fsub_rn(b, kMagic), S.s);
}

// ---------------------------------------------------------------- top-m --

// The M largest keys of a multiset, sorted descending (v[0] largest).  Keys
// are >= 0, so 0 works as the empty value: extra zeros never change the m-th
// largest of a group holding at least m elements.
template <int M>
struct TopM {
    uint32_t v[M];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int i = 0; i < M; ++i) v[i] = 0u;
    }
    __device__ __forceinline__ void insert(uint32_t x) {
#pragma unroll
        for (int i = 0; i < M; ++i) {
            uint32_t hi = max(v[i], x);
            x = min(v[i], x);
            v[i] = hi;
        }
    }
    // Union with another sorted list: the (i+1)-th largest of the union is
    // max(a[i], b[i], max over j < i of min(a[j], b[i-1-j])).
    __device__ __forceinline__ void merge(const uint32_t* b) {
        uint32_t r[M];
#pragma unroll
        for (int i = 0; i < M; ++i) {
            uint32_t x = max(v[i], b[i]);
#pragma unroll
            for (int j = 0; j < i; ++j) x = max(x, min(v[j], b[i - 1 - j]));
            r[i] = x;
        }
#pragma unroll
        for (int i = 0; i < M; ++i) v[i] = r[i];
    }
    __device__ __forceinline__ void warp_reduce() {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            uint32_t o[M];
#pragma unroll
            for (int i = 0; i < M; ++i) o[i] = __shfl_xor_sync(0xFFFFFFFFu, v[i], off);
            merge(o);
        }
    }
};

// ---------------------------------------------------------------- teams --

// A team is TW warps working on one row.  TW == 1: the warp itself; TW == the
// whole block: __syncthreads; otherwise a named barrier per team.
template <int TW, int BLOCK_WARPS>
__device__ __forceinline__ void team_sync(int team) {
    if constexpr (TW == 1) {
        __syncwarp();
    } else if constexpr (TW == BLOCK_WARPS) {
        __syncthreads();
    } else {
        asm volatile("bar.sync %0, %1;" ::"r"(team + 1), "r"(TW * 32) : "memory");
    }
}

}  // namespace gq
