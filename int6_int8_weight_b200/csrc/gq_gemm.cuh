// gq_gemm.cuh -- the consuming GEMM with the dequant fused into its weight
// load: Y[M, N] (+)= X[M, K] * W_hat[N, K]^T on the 5th-generation tensor
// cores, where W_hat[n, k] = bf16(RN(q[n, k] * s[n])) is rebuilt from the
// packed int6 / int8 codes and binary16 row scales of an export while the
// weight tile is staged in shared memory (the fake-quant weights of the
// forward pass, "STE QAT" on "SubSixteen v2" and PR #1202, consumed where
// the GEMM loads them instead of being written out and read back).
//
// One CTA per 128 x 128 output tile and K slice (split K for a small M):
//   warp 0      one lane loads the X tiles by TMA (SWIZZLE_128B, K-major)
//   warp 1      owns the TMEM accumulator (128 lanes x 128 fp32 columns);
//               one lane issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32,
//               M 128, N 128, K 16) and commits each stage back to its
//               producers
//   warps 2..5  dequantize one weight row each per stage into the same
//               SWIZZLE_128B K-major layout, then read the accumulator out
//               of TMEM (tcgen05.ld) and add it into Y
// Stages of (X tile 16 KB + W tile 16 KB) form a ring with mbarriers: full
// X (TMA transaction bytes), full W (128 producer arrivals), empty (the MMA
// commit).  Every wait is bounded by %globaltimer.
#pragma once

#include <cuda.h>
#include "gq_device.cuh"

namespace gq {

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 128;
constexpr int kGemmBK = 64;                              // one 128-byte swizzle row of bf16
constexpr int kGemmStages = 6;
constexpr int kGemmThreads = 192;
constexpr int kGemmTileBytes = kGemmBM * kGemmBK * 2;    // 16 KB, X and W tiles alike
constexpr int kGemmStageBytes = 2 * kGemmTileBytes;
constexpr int kGemmSmemBytes = kGemmStages * kGemmStageBytes + 1024 /* alignment */ + 256 /* barriers */;
constexpr uint32_t kGemmTmemCols = 128;
constexpr unsigned long long kGemmWaitNs = 4000000000ull;

struct GemmParams {
    CUtensorMap tmap_x;          // X [M, K] bf16, box 64 x 128, SWIZZLE_128B
    const uint8_t* packed;       // [N, prb] codes (int6: 4 in 3 bytes; int8: one byte)
    const uint16_t* scale;       // [N] binary16 row scales
    float* y;                    // [M, ldy] fp32, added into (split K) or stored
    int32_t* status;             // nullable: GQ_STATUS_TIMEOUT on an expired wait
    int64_t M, N, K, prb, ldy;
    int32_t qbits;
    int32_t k_tiles;             // 64-wide K tiles of one split
    int32_t accumulate;          // 1: red.add into Y (split K), 0: store
    int32_t pad;
};

// ------------------------------------------------------------- PTX glue --

__device__ __forceinline__ uint32_t g_smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long g_now() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ bool g_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait for the completion of the phase with the given parity.
__device__ __forceinline__ bool g_wait(uint32_t bar, uint32_t parity) {
    if (g_try_wait(bar, parity)) return true;
    const unsigned long long t0 = g_now();
    for (uint32_t i = 1;; ++i) {
        if (g_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0u && g_now() - t0 > kGemmWaitNs) return false;
    }
}

__device__ __forceinline__ void g_bar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void g_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void g_arrive_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// 2-D tiled TMA load (no multicast) of box {x, y} into this CTA's shared memory.
__device__ __forceinline__ void g_tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor: K-major, SWIZZLE_128B, 8-row groups
// 1024 bytes apart (stride byte offset), leading byte offset 16 (unused by
// the swizzled K-major form), descriptor version 1.
__device__ __forceinline__ uint64_t g_smem_desc(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major,
// N = kGemmBN, M = kGemmBM.
constexpr uint32_t kGemmIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kGemmBN >> 3) << 17) |
                                ((uint32_t)(kGemmBM >> 4) << 24);

__device__ __forceinline__ void g_mma(uint32_t tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
        "l"(adesc), "l"(bdesc), "r"(kGemmIdesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void g_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// ------------------------------------------------------------- dequant --

__device__ __forceinline__ uint32_t g_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// One weight row of a stage: 64 codes starting at code k0 of row n, as
// bf16(RN(q * s)) in the K-major SWIZZLE_128B layout (16-byte chunk c of
// row r at chunk position c ^ (r & 7) of the row's 128 bytes).
__device__ __forceinline__ void g_dequant_row(const GemmParams& P, int64_t n, int64_t k0, uint32_t row_addr,
                                              int r) {
    uint32_t code_bits[16];          // int6: 12 words used; int8: 16
    float s = 0.0f;
    if (n < P.N) {
        s = __half2float(__ushort_as_half(P.scale[n]));
        const uint8_t* src = P.packed + n * P.prb + (P.qbits == 6 ? (k0 / 4) * 3 : k0);
        const uint4* v = reinterpret_cast<const uint4*>(src);
        const int nv = P.qbits == 6 ? 3 : 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 u = i < nv ? __ldg(v + i) : make_uint4(0u, 0u, 0u, 0u);
            code_bits[4 * i + 0] = u.x;
            code_bits[4 * i + 1] = u.y;
            code_bits[4 * i + 2] = u.z;
            code_bits[4 * i + 3] = u.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) code_bits[i] = 0u;   // rows past N: zero weights
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {                          // 8 chunks of 8 codes
        float w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int k = 8 * c + j;
            int q;
            if (P.qbits == 6) {
                const int bit = 6 * k;                     // 4 codes per 24 bits = 6 bits each
                const uint32_t lo = code_bits[bit >> 5];
                const uint32_t hi = code_bits[(bit >> 5) + 1 < 16 ? (bit >> 5) + 1 : 15];
                const uint32_t f = __funnelshift_r(lo, hi, bit & 31) & 63u;
                q = (int)(f << 26) >> 26;                  // 6-bit two's complement
            } else {
                q = (int)(int8_t)(code_bits[k >> 2] >> (8 * (k & 3)));
            }
            w[j] = __fmul_rn((float)q, s);
        }
        const uint4 out = make_uint4(g_bf16x2(w[0], w[1]), g_bf16x2(w[2], w[3]), g_bf16x2(w[4], w[5]),
                                     g_bf16x2(w[6], w[7]));
        const uint32_t dst = row_addr + (uint32_t)((c ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(out.x), "r"(out.y), "r"(out.z),
                     "r"(out.w)
                     : "memory");
    }
}

// ----------------------------------------------------------------- kernel --

__global__ void __launch_bounds__(kGemmThreads, 1) gemm_dequant_kernel(const __grid_constant__ GemmParams P) {
    extern __shared__ unsigned char g_smem[];
    const uint32_t raw = g_smem_u32(g_smem);
    const uint32_t base = (raw + 1023u) & ~1023u;          // SWIZZLE_128B tiles: 1024-byte aligned
    const uint32_t bars = base + kGemmStages * kGemmStageBytes;
    auto full_x = [&](int s) { return bars + 8u * (uint32_t)s; };
    auto full_w = [&](int s) { return bars + 8u * (uint32_t)(kGemmStages + s); };
    auto empty = [&](int s) { return bars + 8u * (uint32_t)(2 * kGemmStages + s); };
    const uint32_t done = bars + 8u * (uint32_t)(3 * kGemmStages);
    const uint32_t tmem_slot = done + 8u;
    auto x_tile = [&](int s) { return base + (uint32_t)s * kGemmStageBytes; };
    auto w_tile = [&](int s) { return base + (uint32_t)s * kGemmStageBytes + kGemmTileBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = (int64_t)blockIdx.x * kGemmBN;
    const int64_t m0 = (int64_t)blockIdx.y * kGemmBM;
    const int kt0 = blockIdx.z * P.k_tiles;
    const int KT = P.k_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            g_bar_init(full_x(s), 1);
            g_bar_init(full_w(s), 128);
            g_bar_init(empty(s), 1);
        }
        g_bar_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tmap_x)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tmem_slot),
                     "r"(kGemmTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    uint32_t tmem;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(tmem) : "r"(tmem_slot) : "memory");

    bool ok = true;
    if (warp == 0) {
        // ------------------------------------------------ X tiles (TMA) --
        if (lane == 0) {
            for (int kt = 0; kt < KT && ok; ++kt) {
                const int s = kt % kGemmStages, k = kt / kGemmStages;
                if (k > 0 && !g_wait(empty(s), (uint32_t)((k - 1) & 1))) ok = false;
                if (!ok) break;
                g_arrive_tx(full_x(s), kGemmTileBytes);
                g_tma_load_2d(x_tile(s), &P.tmap_x, (kt0 + kt) * kGemmBK, (int)m0, full_x(s));
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA --
        if (lane == 0) {
            for (int kt = 0; kt < KT && ok; ++kt) {
                const int s = kt % kGemmStages, k = kt / kGemmStages;
                const uint32_t par = (uint32_t)(k & 1);
                if (!g_wait(full_x(s), par) || !g_wait(full_w(s), par)) {
                    ok = false;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
                for (int kk = 0; kk < kGemmBK / 16; ++kk)
                    g_mma(tmem, g_smem_desc(x_tile(s) + 32u * kk), g_smem_desc(w_tile(s) + 32u * kk),
                          (kt > 0 || kk > 0) ? 1u : 0u);
                g_commit(empty(s));
            }
            g_commit(done);              // also after a failure: lets the epilogue go
        }
    } else {
        // ------------------------------------ W tiles (dequant), epilogue --
        const int r = threadIdx.x - 64;                    // weight row of the tile, 0..127
        for (int kt = 0; kt < KT && ok; ++kt) {
            const int s = kt % kGemmStages, k = kt / kGemmStages;
            if (k > 0 && !g_wait(empty(s), (uint32_t)((k - 1) & 1))) ok = false;
            if (!ok) break;
            g_dequant_row(P, n0 + r, (int64_t)(kt0 + kt) * kGemmBK, w_tile(s) + 128u * (uint32_t)r, r);
            // generic-proxy writes -> visible to the tensor core (async proxy)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            g_arrive(full_w(s));
        }
        if (!g_wait(done, 0u)) ok = false;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const int quarter = warp & 3;                      // TMEM lanes this warp may read
        const int64_t m = m0 + 32 * quarter + lane;
        for (int c = 0; c < kGemmBN / 16; ++c) {
            uint32_t v[16];
            const uint32_t taddr = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(16 * c);
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                "%13, %14, %15}, [%16];"
                : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                  "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                  "=r"(v[15])
                : "r"(taddr));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            if (m < P.M && ok) {
                float* yrow = P.y + m * P.ldy + n0 + 16 * c;
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const int64_t col = n0 + 16 * c + j;
                    if (col + 3 < P.N) {
                        if (P.accumulate) {
                            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(yrow + j),
                                         "f"(__uint_as_float(v[j])), "f"(__uint_as_float(v[j + 1])),
                                         "f"(__uint_as_float(v[j + 2])), "f"(__uint_as_float(v[j + 3]))
                                         : "memory");
                        } else {
                            *reinterpret_cast<float4*>(yrow + j) =
                                make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                            __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
                        }
                    } else {
                        for (int e = 0; e < 4 && col + e < P.N; ++e) {   // the last columns of Y
                            if (P.accumulate) atomicAdd(yrow + j + e, __uint_as_float(v[j + e]));
                            else yrow[j + e] = __uint_as_float(v[j + e]);
                        }
                    }
                }
            }
        }
    }
    if (!ok && lane == 0 && P.status) atomicOr(reinterpret_cast<unsigned int*>(P.status), 0x4u);
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kGemmTmemCols)
                     : "memory");
    }
}

}  // namespace gq
