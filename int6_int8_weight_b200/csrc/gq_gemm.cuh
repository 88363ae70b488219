// gq_gemm.cuh -- the consuming GEMM with the dequant fused into its weight
// load: Y[M, N] (+)= X[M, K] * W_hat[N, K]^T on the 5th-generation tensor
// cores, where W_hat[n, k] = bf16(RN(q[n, k] * s[n])) is rebuilt from the
// packed int6 / int8 codes and binary16 row scales of an export while the
// weight tile is staged in shared memory (the fake-quant weights of the
// forward pass, "STE QAT" on "SubSixteen v2" and PR #1202, consumed where
// the GEMM loads them instead of being written out and read back).
//
// One CTA per output tile and K slice (split K for a small M).  For M > 128
// the tile is 128 tokens x 128 weight rows (A = X, B = W_hat); for M <= 128
// the operands swap (A = W_hat, 128 weight rows; B = X, nt = 16 .. 128 token
// rows), so a small batch does not pay for 128-row MMAs on padding.
//   warp 0        one lane loads the X tiles by TMA (SWIZZLE_128B, K-major)
//   warp 1        one lane loads the packed code tiles by TMA, far ahead
//   warps 2, 3    issue tcgen05.mma (kind::f16, bf16 x bf16 -> fp32, M 128,
//                 K 16), stage kt by warp 2 + kt % 2 into accumulator kt % 2
//   warps 4..19   dequantize, in two groups of 8 warps (stage kt by group
//                 kt % 2, two threads per weight row), from the staged codes
//                 into the SWIZZLE_128B K-major layout; then all 16 read the
//                 accumulators out of TMEM (tcgen05.ld, four warps per lane
//                 quarter), add them and store or add the sums into Y
// A stage is one 64-wide swizzle atom of K (4 MMAs).  Every hand-off
// between warps costs a few hundred ns of latency, so the work alternates
// between two MMA warps and two dequant groups, and the rings (W_hat,
// X and codes, each with its own depth) are deep enough that a slot's
// round trip (dequant -> MMA -> commit -> dequant) overlaps the next
// stages.  The MMA warp waits for the stage's X tile (TMA bytes) and
// W_hat tile (the 256 arrivals of its dequant group); the stage's one
// commit (on a ring of its own) frees both slots.  Every wait is bounded
// by %globaltimer.
#pragma once

#include <cuda.h>
#include "gq_device.cuh"

namespace gq {

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 128;
constexpr int kGemmBK = 64;                              // a stage: one 128-byte swizzle atom of bf16 along K
constexpr int kGemmWStagesMax = 8;                       // W_hat ring
constexpr int kGemmXStagesMax = 14;                      // X ring
constexpr int kGemmDoneRing = 32;                        // per-stage MMA commits (> twice either depth)
constexpr int kGemmCStagesMax = 12;                      // code ring
constexpr int kGemmMmaWarps = 2;                         // stage kt is issued by MMA warp kt % 2
constexpr int kGemmDqGroups = 2;                         // stage kt is dequantized by group kt % 2
constexpr int kGemmGroup = 2 * kGemmBN;                  // threads of a group: two per weight row
constexpr int kGemmDequant = kGemmDqGroups * kGemmGroup;
constexpr int kGemmDqWarp0 = 2 + kGemmMmaWarps;          // first dequant warp
constexpr int kGemmThreads = 32 * kGemmDqWarp0 + kGemmDequant;
constexpr int kGemmAtomBytes = kGemmBN * kGemmBK * 2;    // 16 KB: 128 rows x 64 bf16
constexpr int kGemmBarBytes = 1024;
constexpr int kGemmSmemBytes = 232448;                   // all of it: 227 KB
constexpr int kGemmRingBytes = kGemmSmemBytes - 1024 /* alignment */ - kGemmBarBytes;
constexpr unsigned long long kGemmWaitNs = 4000000000ull;
static_assert(kGemmDoneRing % kGemmMmaWarps == 0 && kGemmDoneRing % kGemmDqGroups == 0, "commit ring");
static_assert(2 * kGemmWStagesMax < kGemmDoneRing && 2 * kGemmXStagesMax < kGemmDoneRing, "commit ring depth");

struct GemmParams {
    CUtensorMap tmap_x;          // X [M, K] bf16, box 64 x nt, SWIZZLE_128B
    CUtensorMap tmap_w;          // codes [N, prb] bytes, box (64 codes' bytes) x 128, no swizzle
    const uint16_t* scale;       // [N] binary16 row scales
    float* y;                    // [M, ldy] fp32, added into (split K) or stored
    int32_t* status;             // nullable: GQ_STATUS_TIMEOUT on an expired wait
    int64_t M, N, K, ldy;
    int32_t qbits;
    int32_t k_stages;            // 64-wide K stages in all
    int32_t splits;              // K splits (grid z); split z takes a contiguous run of stages
    int32_t accumulate;          // 1: red.add into Y (split K), 0: store
    int32_t swap;                // 1: A = W_hat, B = X (M <= 128)
    int32_t nt;                  // token rows of an X tile (128, or 16 .. 128 swapped)
    uint32_t idesc;              // tcgen05 instruction descriptor of the tile's MMA
    uint32_t tmem_cols;          // TMEM columns allocated: kGemmMmaWarps accumulators
    uint32_t acc_cols;           // columns of one accumulator (a power of two >= 32)
    int32_t w_stages;            // ring depths
    int32_t x_stages;
    int32_t c_stages;
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

// Test for the completion of the phase with the given parity; the thread
// may sleep in the barrier for up to the hint (100 us) while it waits, so
// that waiting warps leave the issue slots to the working ones.
__device__ __forceinline__ bool g_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(100000u)
        : "memory");
    return done != 0;
}

// Bounded wait for the completion of the phase with the given parity.
__device__ __forceinline__ bool g_wait(uint32_t bar, uint32_t parity) {
    if (g_try_wait(bar, parity)) return true;
    const unsigned long long t0 = g_now();
    for (;;) {
        if (g_try_wait(bar, parity)) return true;
        if (g_now() - t0 > kGemmWaitNs) return false;
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
// M rows of A (64 / 128), N rows of B (a multiple of 16, 16 .. 256).
__host__ __device__ constexpr uint32_t gemm_idesc(uint32_t m, uint32_t n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

// One elected lane of a converged warp.
__device__ __forceinline__ bool g_elect() {
    uint32_t e;
    asm volatile(
        "{\n .reg .pred e;\n"
        " elect.sync _|e, 0xffffffff;\n"
        " selp.u32 %0, 1, 0, e;\n}"
        : "=r"(e));
    return e != 0;
}

// g_wait by every lane of a warp, with a warp-uniform result.
__device__ __forceinline__ bool g_wait_warp(uint32_t bar, uint32_t parity) {
    return __all_sync(0xffffffffu, g_wait(bar, parity));
}

// The 4 MMAs (K = 16 each) of one stage, issued by one elected lane of
// the (converged) calling warp from a single asm block: nothing runs
// between them in the issuing thread, which keeps the tensor pipe fed
// (scalar work between consecutive tcgen05.mma roughly halves the issue
// rate).  The first MMA into an accumulator overwrites it (accumulate = 0).
__device__ __forceinline__ void g_mma_stage(uint32_t tmem, const uint64_t (&a)[4], const uint64_t (&b)[4],
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %9, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %5, %10, p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %10, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %10, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %10, 1;\n\t"
        "}\n" ::"r"(tmem),
        "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "r"(accumulate),
        "r"(idesc)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far is done (one
// elected lane of the calling warp commits).
__device__ __forceinline__ void g_commit(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(bar)
        : "memory");
}

// 16 consecutive accumulator columns of this thread's TMEM lane, summed
// over the `nacc` accumulators `stride` columns apart (in accumulator order).
__device__ __forceinline__ void g_acc16(uint32_t taddr, uint32_t stride, int nacc, float (&f)[16]) {
    for (int a = 0; a < nacc; ++a) {
        uint32_t v[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
            "%12, %13, %14, %15}, [%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(taddr + (uint32_t)a * stride));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int i = 0; i < 16; ++i) f[i] = a == 0 ? __uint_as_float(v[i]) : __fadd_rn(f[i], __uint_as_float(v[i]));
    }
}

// ------------------------------------------------------------- dequant --

__device__ __forceinline__ uint32_t g_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Two binary32 lanes in one 64-bit register (paired .rn f32x2 arithmetic).
__device__ __forceinline__ uint64_t g_f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

// Per-row constants of the dequant.  A code field with its top bit inverted
// (two's complement -> offset binary, u = q + 2^(bits-1)) and placed at bit
// p of a word under the exponent of 2^23 reads as the float
// F = 2^23 + u * 2^p, so that
//     q * s = F * S_p - C_p * S_p,   S_p = s * 2^-p,  C_p = 2^23 + 2^(bits-1) * 2^p,
// one fused multiply-add per code, exact: q * s has at most 8 + 11
// significant bits, S_p is s scaled by a power of two, and C_p * S_p is
// exact because C_p has at most 13 significant bits (p >= 6 for int6,
// p >= 4 for int8) against the 11 of a binary16 s.  The only rounding is
// the final one to bf16.  int6 takes fields at p = 12 and p = 6 (two codes
// per 12-bit view of the code stream), int8 at p = 8, 4 and 12.
struct GDeq {
    uint64_t s_a, c_a;           // int6 (S12, S6) / int8 even pair (S8, S8), and -C_p * S_p
    uint64_t s_b, c_b;           // int8 odd pair (S4, S12)
};

__device__ __forceinline__ GDeq g_deq_consts(int qbits, float s) {
    auto sp = [&](int p) { return __fmul_rn(s, __int_as_float((127 - p) << 23)); };      // s * 2^-p
    auto cs = [&](int bits, int p) {                                                    // -C_p * S_p
        return __fmul_rn(-(8388608.0f + (float)(1 << (bits - 1 + p))), sp(p));
    };
    GDeq d;
    if (qbits == 6) {
        d.s_a = g_f2(sp(12), sp(6));
        d.c_a = g_f2(cs(6, 12), cs(6, 6));
        d.s_b = d.c_b = 0;
    } else {
        d.s_a = g_f2(sp(8), sp(8));
        d.c_a = g_f2(cs(8, 8), cs(8, 8));
        d.s_b = g_f2(sp(4), sp(12));
        d.c_b = g_f2(cs(8, 4), cs(8, 12));
    }
    return d;
}

// The field of `v` at bits p .. p + bits - 1 (mask m), top bit inverted,
// under the exponent of 2^23 (x = inverted bit | 0x4B000000): one LOP3.
__device__ __forceinline__ float g_field(uint32_t v, uint32_t m, uint32_t x) {
    return __uint_as_float(((v ^ x) & m) | (x & ~m));
}

__device__ __forceinline__ uint32_t g_pair_bf16(float f0, float f1, uint64_t s2, uint64_t c2) {
    uint64_t w2;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(w2) : "l"(g_f2(f0, f1)), "l"(s2), "l"(c2));
    float w0, w1;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(w0), "=f"(w1) : "l"(w2));
    return g_bf16x2(w0, w1);
}

// Half a stage of one weight row: 32 codes (half of the swizzle atom,
// chunks 4h .. 4h + 3) staged at `codes` (the code stage is released on
// `release` once they are used), as bf16(RN(q * s)) into the K-major
// SWIZZLE_128B layout (16-byte chunk c of row r at chunk position c ^ (r & 7)
// of the row's 128 bytes at `row_addr`).
template <int QBITS>
__device__ __forceinline__ void g_dequant_part(uint32_t codes, uint32_t release, uint32_t row_addr, int r, int h,
                                               const GDeq& d) {
    uint32_t w[8];                                         // int6: 6 words (+1 zero); int8: 8 words
    if constexpr (QBITS == 6) {
#pragma unroll
        for (int i = 0; i < 3; ++i)                        // 24 bytes, 8-byte aligned
            asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];"
                         : "=r"(w[2 * i]), "=r"(w[2 * i + 1])
                         : "r"(codes + 8u * i)
                         : "memory");
        w[6] = 0u;
    } else {
#pragma unroll
        for (int i = 0; i < 2; ++i)
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[4 * i]), "=r"(w[4 * i + 1]), "=r"(w[4 * i + 2]), "=r"(w[4 * i + 3])
                         : "r"(codes + 16u * i)
                         : "memory");
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {                          // 4 chunks of 8 codes
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = 4 * c + j;                       // codes 2i and 2i + 1
            if constexpr (QBITS == 6) {
                // the code stream shifted right by 12 (i - 1) holds code 2i at
                // bit 12; shifted by 12 i it holds code 2i + 1 at bit 6
                const int sh = 12 * i;
                const uint32_t vb = __funnelshift_r(w[sh >> 5], w[(sh >> 5) + 1], sh & 31);
                uint32_t va;
                if (i == 0) {
                    va = w[0] << 12;
                } else {
                    const int sa = sh - 12;
                    va = __funnelshift_r(w[sa >> 5], w[(sa >> 5) + 1], sa & 31);
                }
                out[j] = g_pair_bf16(g_field(va, 0x3F000u, 0x4B020000u), g_field(vb, 0xFC0u, 0x4B000800u), d.s_a,
                                     d.c_a);
            } else {
                const uint32_t wd = w[i >> 1];
                if ((i & 1) == 0) {                        // bytes 0, 1: both at bit 8
                    out[j] = g_pair_bf16(g_field(wd << 8, 0xFF00u, 0x4B008000u), g_field(wd, 0xFF00u, 0x4B008000u),
                                         d.s_a, d.c_a);
                } else {                                   // bytes 2, 3: at bits 4 and 12 of wd >> 12
                    const uint32_t v = wd >> 12;
                    out[j] = g_pair_bf16(g_field(v, 0xFF0u, 0x4B000800u), g_field(v, 0xFF000u, 0x4B080000u), d.s_b,
                                         d.c_b);
                }
            }
        }
        const uint32_t dst = row_addr + (uint32_t)(((4 * h + c) ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(out[0]), "r"(out[1]), "r"(out[2]),
                     "r"(out[3])
                     : "memory");
    }
    // The code slot is released only now that every loaded word has been
    // used: an arrive issued while a shared load is still in flight lets the
    // next TMA copy (async proxy) overwrite the slot before the load reads
    // it, and the release order of the arrive does not cover that.
    g_arrive(release);
}

// ----------------------------------------------------------------- kernel --

__global__ void __launch_bounds__(kGemmThreads, 1) gemm_dequant_kernel(const __grid_constant__ GemmParams P) {
    extern __shared__ unsigned char g_smem[];
    const uint32_t raw = g_smem_u32(g_smem);
    const uint32_t base = (raw + 1023u) & ~1023u;          // SWIZZLE_128B tiles: 1024-byte aligned
    // [W_hat ring][X ring][code ring: 128 rows x 48 | 64 bytes][barriers]
    const int DW = P.w_stages, DX = P.x_stages, DC = P.c_stages;
    const uint32_t x_bytes = (uint32_t)P.nt * 128u;
    const uint32_t row_code_bytes = P.qbits == 6 ? 48u : 64u;        // 64 codes of a row
    const uint32_t xs0 = base + (uint32_t)DW * kGemmAtomBytes;
    const uint32_t cs0 = xs0 + (uint32_t)DX * x_bytes;
    const uint32_t bars = base + (uint32_t)(kGemmSmemBytes - 1024 - kGemmBarBytes);
    auto full_w = [&](int s) { return bars + 8u * (uint32_t)s; };                      // a group's arrivals
    auto full_x = [&](int s) { return bars + 8u * (uint32_t)(kGemmWStagesMax + s); };  // X TMA bytes
    auto mma_done = [&](int kt) {                                                      // stage kt's commit
        return bars + 8u * (uint32_t)(kGemmWStagesMax + kGemmXStagesMax + kt % kGemmDoneRing);
    };
    constexpr int kCBar = kGemmWStagesMax + kGemmXStagesMax + kGemmDoneRing;
    auto full_c = [&](int s) { return bars + 8u * (uint32_t)(kCBar + s); };
    auto empty_c = [&](int s) { return bars + 8u * (uint32_t)(kCBar + kGemmCStagesMax + s); };
    const uint32_t done = bars + 8u * (uint32_t)(kCBar + 2 * kGemmCStagesMax);
    const uint32_t tmem_slot = done + 8u;
    auto w_tile = [&](int s) { return base + (uint32_t)s * kGemmAtomBytes; };
    auto x_tile = [&](int s) { return xs0 + (uint32_t)s * x_bytes; };
    auto c_tile = [&](int s) { return cs0 + (uint32_t)s * (kGemmBN * row_code_bytes); };
    // parity of stage kt's commit on its done barrier
    auto done_parity = [&](int kt) { return (uint32_t)((kt / kGemmDoneRing) & 1); };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = (int64_t)blockIdx.x * kGemmBN;
    const int64_t m0 = (int64_t)blockIdx.y * P.nt;
    const int kbase = P.k_stages / P.splits, kextra = P.k_stages % P.splits;
    const int KT = kbase + ((int)blockIdx.z < kextra ? 1 : 0);
    const int kt0 = (int)blockIdx.z * kbase + min((int)blockIdx.z, kextra);

    if (threadIdx.x == 0) {
        for (int s = 0; s < DW; ++s) g_bar_init(full_w(s), kGemmGroup);
        for (int s = 0; s < DX; ++s) g_bar_init(full_x(s), 1);
        for (int s = 0; s < kGemmDoneRing; ++s) g_bar_init(mma_done(s), 1);
        for (int s = 0; s < DC; ++s) {
            g_bar_init(full_c(s), 1);
            g_bar_init(empty_c(s), kGemmGroup);
        }
        g_bar_init(done, kGemmMmaWarps);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tmap_x)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tmap_w)) : "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tmem_slot),
                     "r"(P.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    uint32_t tmem;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(tmem) : "r"(tmem_slot) : "memory");

    bool ok = true;
    // The control warps run their loops with all 32 lanes (the waits and
    // the descriptor arithmetic stay warp-uniform); one elected lane issues
    // each copy, MMA and commit.
    const bool leader = g_elect();
    if (warp == 0) {
        // ------------------------------------------------ X tiles (TMA) --
        int issued = 0;
        for (int kt = 0; kt < KT && ok; ++kt) {
            const int s = kt % DX;
            // the slot's previous stage has been consumed by its MMAs
            if (kt >= DX && !g_wait_warp(mma_done(kt - DX), done_parity(kt - DX))) ok = false;
            if (!ok) break;
            if (leader) {
                g_arrive_tx(full_x(s), x_bytes);
                g_tma_load_2d(x_tile(s), &P.tmap_x, (kt0 + kt) * kGemmBK, (int)m0, full_x(s));
            }
            issued = kt + 1;
        }
        // no copy may still be landing when the CTA leaves (instant unless a wait expired)
        for (int kt = max(0, issued - DX); kt < issued; ++kt)
            if (!g_wait_warp(full_x(kt % DX), (uint32_t)((kt / DX) & 1))) ok = false;
    } else if (warp == 1) {
        // --------------------------------------------- code tiles (TMA) --
        int issued = 0;
        for (int kt = 0; kt < KT && ok; ++kt) {
            const int s = kt % DC, g = kt / DC;
            if (g > 0 && !g_wait_warp(empty_c(s), (uint32_t)((g - 1) & 1))) ok = false;
            if (!ok) break;
            if (leader) {
                g_arrive_tx(full_c(s), kGemmBN * row_code_bytes);   // out-of-range rows are zero-filled
                g_tma_load_2d(c_tile(s), &P.tmap_w, (kt0 + kt) * (int)row_code_bytes, (int)n0, full_c(s));
            }
            issued = kt + 1;
        }
        for (int kt = max(0, issued - DC); kt < issued; ++kt)
            if (!g_wait_warp(full_c(kt % DC), (uint32_t)((kt / DC) & 1))) ok = false;
    } else if (warp < kGemmDqWarp0) {
        // ------------------------------------------------------- MMA --
        // MMA warp j issues stages j, j + 2, ... into accumulator j: the
        // issuing thread's serial latency (barrier wait, descriptors,
        // commit) is shared between the warps, and the tensor pipe takes
        // their MMAs as they come
        const int j = warp - 2;
        const uint32_t acc = tmem + (uint32_t)j * P.acc_cols;
        for (int kt = j; kt < KT && ok; kt += kGemmMmaWarps) {
            const int s = kt % DW, sx = kt % DX;
            // the stage's X tile (TMA) and W_hat tile (dequant) are in place
            if (!g_wait_warp(full_x(sx), (uint32_t)((kt / DX) & 1)) ||
                !g_wait_warp(full_w(s), (uint32_t)((kt / DW) & 1))) {
                ok = false;
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            // descriptors of the stage's K = 16 steps: 32 bytes apart within the swizzle atom
            uint64_t da[4], db[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint64_t dx = g_smem_desc(x_tile(sx) + 32u * (uint32_t)i);
                const uint64_t dw = g_smem_desc(w_tile(s) + 32u * (uint32_t)i);
                da[i] = P.swap ? dw : dx;
                db[i] = P.swap ? dx : dw;
            }
            g_mma_stage(acc, da, db, P.idesc, kt >= kGemmMmaWarps ? 1u : 0u);
            g_commit(mma_done(kt));      // frees the stage's X and W_hat slots once these MMAs are done
        }
        g_commit(done);                  // also after a failure: lets the epilogue go
    } else {
        // ------------------------------------ W_hat tiles (dequant), epilogue --
        // group gi takes stages gi, gi + 2, ...; two threads per weight row,
        // the 8 lanes of a quarter warp on 8 consecutive rows with the same
        // half (conflict-free swizzled stores)
        const int t = threadIdx.x - 32 * kGemmDqWarp0;
        const int gi = t / kGemmGroup, tg = t % kGemmGroup;
        const int r = 8 * (tg >> 4) + (tg & 7), h = (tg >> 3) & 1;
        const float srow = n0 + r < P.N ? __half2float(__ushort_as_half(P.scale[n0 + r])) : 0.0f;
        const GDeq deq = g_deq_consts(P.qbits, srow);
        const uint32_t code_off = row_code_bytes * (uint32_t)r + (row_code_bytes / 2u) * (uint32_t)h;
        for (int kt = gi; kt < KT && ok; kt += kGemmDqGroups) {
            const int s = kt % DW;
            const int cs = kt % DC, g = kt / DC;
            // the codes have landed; the slot's previous stage has been consumed
            if (!g_wait(full_c(cs), (uint32_t)(g & 1)) ||
                (kt >= DW && !g_wait(mma_done(kt - DW), done_parity(kt - DW)))) {
                ok = false;
                break;
            }
            const uint32_t dst = w_tile(s) + 128u * (uint32_t)r;
            if (P.qbits == 6) g_dequant_part<6>(c_tile(cs) + code_off, empty_c(cs), dst, r, h, deq);
            else g_dequant_part<8>(c_tile(cs) + code_off, empty_c(cs), dst, r, h, deq);
            // generic-proxy writes -> visible to the tensor core (async proxy)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            g_arrive(full_w(s));
        }
        if (!g_wait(done, 0u)) ok = false;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const int quarter = warp & 3;                      // TMEM lanes this warp may read
        const int cpart = (warp - kGemmDqWarp0) >> 2;      // four warps per lane quarter
        const int nacc = min(KT, kGemmMmaWarps);           // accumulators holding a partial sum
        if (P.swap) {
            // accumulator lane = weight row n, column = token m0 + j
            const int64_t n = n0 + 32 * quarter + lane;
            for (int c = cpart; c < P.nt / 16; c += 4) {
                float v[16];
                g_acc16(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(16 * c), P.acc_cols, nacc, v);
                if (n < P.N && ok) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int64_t m = m0 + 16 * c + j;
                        if (m < P.M) {
                            float* dst = P.y + m * P.ldy + n;   // a warp writes 32 consecutive floats
                            if (P.accumulate) atomicAdd(dst, v[j]);
                            else *dst = v[j];
                        }
                    }
                }
            }
        } else {
            // accumulator lane = token m, column = weight row n0 + j
            const int64_t m = m0 + 32 * quarter + lane;
            for (int c = cpart * (kGemmBN / 64); c < (cpart + 1) * (kGemmBN / 64); ++c) {
                float v[16];
                g_acc16(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(16 * c), P.acc_cols, nacc, v);
                if (m < P.M && ok) {
                    float* yrow = P.y + m * P.ldy + n0 + 16 * c;
#pragma unroll
                    for (int j = 0; j < 16; j += 4) {
                        const int64_t col = n0 + 16 * c + j;
                        if (col + 3 < P.N) {
                            if (P.accumulate) {
                                asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(yrow + j),
                                             "f"(v[j]), "f"(v[j + 1]),
                                             "f"(v[j + 2]), "f"(v[j + 3])
                                             : "memory");
                            } else {
                                *reinterpret_cast<float4*>(yrow + j) =
                                    make_float4(v[j], v[j + 1],
                                                v[j + 2], v[j + 3]);
                            }
                        } else {
                            for (int e = 0; e < 4 && col + e < P.N; ++e) {   // the last columns of Y
                                if (P.accumulate) atomicAdd(yrow + j + e, v[j + e]);
                                else yrow[j + e] = v[j + e];
                            }
                        }
                    }
                }
            }
        }
    }
    if (!ok && lane == 0 && P.status) atomicOr(reinterpret_cast<unsigned int*>(P.status), 0x4u);
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 2) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(P.tmem_cols)
                     : "memory");
    }
}

}  // namespace gq
