// gq_gemm.cuh -- the consuming GEMM with the dequant fused into its weight
// load: Y[M, N] = X[M, K] * W_hat[N, K]^T on the 5th-generation tensor cores,
// where W_hat[n, k] = bf16(RN(q[n, k] * s[n])) is rebuilt from the packed
// int6 / int8 codes and binary16 row scales of an export (the fake-quant
// weights of the forward pass, "STE QAT" on "SubSixteen v2" and PR #1202,
// consumed where the GEMM loads them instead of being written out and read
// back).
//
// Tile: 128 weight rows x nt tokens (nt = 16 .. 256), K in stages of 64.
// The operands are swapped so that the weight tile is the MMA's A operand
// (M = 128) and the token tile its B operand (N = nt):
//   - W_hat never touches shared memory: the dequant threads write it into
//     tensor memory with tcgen05.st (thread r of a lane quarter owns weight
//     row r of the tile), and tcgen05.mma reads A from there.  A 64-wide
//     stage of W_hat is 32 TMEM columns (two bf16 per 32-bit column);
//   - X tiles arrive by TMA (SWIZZLE_128B, K-major) in shared memory;
//   - the packed codes arrive by TMA (or, for int6 rows whose byte length is
//     not a multiple of 16, by 4-byte cp.async copies) in shared memory.
// Shared memory then only carries codes and X, so the MMA's operand reads do
// not compete with W_hat traffic, and an MMA of a small token tile runs at
// about 40 ns per stage (four K = 16 MMAs) instead of ~120 ns with A staged in
// shared memory.
//
// Persistent blocks, one per SM.  Work is a list of stage units (tile, k
// stage), tile-major: with few tiles (decode-sized batches) the units are
// split evenly over the blocks (stream-K: a block's range crosses tile
// boundaries, every partial sum is added into Y, which is zeroed first);
// otherwise each block takes whole tiles round-robin and stores them.
//
// Chunks.  One thread can start a TMA copy only about every 250 ns, whatever
// its size, so copies move CS consecutive K stages at once (a chunk: CS = 4
// for packed codes; 1 for the fake-quant modes, whose stage of bf16 / fp32
// weights is already 16 / 32 KB): one copy of the code rows (128 rows x
// CS * 48 / 64 bytes) and, per X slot of XS stages (XS = 4, 2, 1 for token
// tiles of <= 64, 128, 256), one copy of the token tile (a 3-D view of X,
// {64, nt, XS} with the 128-byte swizzle, when K % 64 == 0; else one 2-D
// copy per stage).  A chunk is also the unit of the MMA hand-off:
// one issuer runs all of a chunk's stages and commits once.  Chunks are
// aligned to the tile's K stages; a block's first and last chunk of a tile
// may hold only part of their stages (the copies still move the whole chunk).
//
// Warp roles (24 warps):
//   warp 0        code producer (TMA, or 4-byte cp.async copies)
//   warps 1, 2    MMA issuers: chunk c by issuer c % NI (NI = 2 for nt <= 64,
//                 each with its own accumulator; else NI = 1)
//   warp 3        TMEM allocation, then the X producer (TMA)
//   warps 4 .. 7  epilogue: accumulators -> Y (one warp per lane quarter)
//   warps 8 .. 23 dequant, four groups of four warps (one per lane quarter);
//                 group g takes sub-stage g % CS of every (4 / CS)-th chunk
// Every wait is an mbarrier wait bounded by %globaltimer; on expiry the
// waiter records GQ_STATUS_TIMEOUT and its role stops.  Before the block
// exits, the producers wait (bounded) for their copies in flight, the
// issuers for their MMAs, and TMEM is released.
#pragma once

#include <cuda.h>
#include "gq_device.cuh"

namespace gq {

constexpr int kGemmBN = 128;                             // weight rows per tile (the MMA's M)
constexpr int kGemmBK = 64;                              // K per stage
constexpr int kGemmGroups = 4;                           // dequant groups
constexpr int kGemmCSMax = 4;                            // stages per chunk (max)
constexpr int kGemmDq0 = 8;                              // first dequant warp
constexpr int kGemmEpi0 = 4;                             // first epilogue warp
constexpr int kGemmThreads = 32 * (kGemmDq0 + 4 * kGemmGroups);
constexpr int kGemmMaxX = 16;                            // X chunk slots (max)
constexpr int kGemmMaxC = 16;                            // code chunk slots (max)
constexpr int kGemmMaxWS = 16;                           // W_hat stage slots in TMEM (chunk slots x stages, max)
constexpr int kGemmMaxDone = 32;                         // per-chunk MMA commit ring (max)
constexpr int kGemmBarBytes = 8 * (2 * kGemmMaxX + 2 * kGemmMaxC + kGemmMaxWS + kGemmMaxDone + 8) + 64;
constexpr int kGemmSmemBytes = 232448;                   // all of it: 227 KB
constexpr int kGemmRingBytes = kGemmSmemBytes - 1024 /* alignment */ - kGemmBarBytes;
constexpr unsigned long long kGemmWaitNs = 4000000000ull;

struct GemmParams {
    CUtensorMap tmap_x;          // X: 3-D {64, M, K / 64} box {64, nt, CS}, or 2-D [M, K] box {64, nt}; SWIZZLE_128B
    CUtensorMap tmap_w;          // codes [N, prb] bytes, box (CS stages' bytes) x 128, no swizzle (TMA mode)
    const uint8_t* codes;        // packed codes (copy mode)
    const uint16_t* scale;       // [N] binary16 row scales (codes)
    const float* clip;           // [N] row clips (weight modes)
    int32_t wmode;               // 0: packed codes; 1: bf16 weights; 2: fp32 weights (fake-quant on load)
    int32_t w3d;                 // fp32 weights: 1 = one 3-D copy {32, 128, 2} per stage, 0 = two 2-D copies
    int32_t export_scale;        // weight modes: 1 = binary16 row scales, 0 = binary32
    float* y;                    // [M, ldy] fp32
    int32_t* status;             // nullable: GQ_STATUS_TIMEOUT on an expired wait
    int64_t M, N, K, ldy, prb;
    int32_t qbits;
    int32_t code_copy;           // 1: codes by cp.async (prb % 16 != 0), 0: by TMA
    int32_t x3d;                 // 1: one 3-D copy of X per X slot, 0: one 2-D copy per stage
    int32_t cs;                  // stages per chunk (codes, W_hat, MMA commits)
    int32_t xs;                  // stages per X slot (divides cs)
    int32_t kt_per_tile;         // 64-wide K stages per tile
    int32_t tiles_m;             // token tiles
    int64_t tiles;               // tiles_n * tiles_m
    int32_t streamk;             // 1: stage units split evenly, partial sums added; 0: whole tiles
    int32_t nt;                  // tokens per tile (the MMA's N)
    int32_t ni;                  // MMA issuers (accumulators)
    uint32_t idesc;              // tcgen05 instruction descriptor
    uint32_t acc_cols;           // TMEM columns of one accumulator
    int32_t dx, dc, dw, dd;      // ring depths: X slots; chunks of codes, W_hat (TMEM), MMA commits
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

// Test for the completion of the phase with the given parity; a thread that
// finds it incomplete may be suspended in the barrier for up to the hint
// (20 us) until it completes, so that waiting warps leave the issue slots to
// the working ones (24 warps share four schedulers).
__device__ __forceinline__ bool g_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(20000u)
        : "memory");
    return done != 0;
}

// Bounded wait for the completion of the phase with the given parity.
__device__ __forceinline__ bool g_wait(uint32_t bar, uint32_t parity) {
    if (g_try_wait(bar, parity)) return true;
    const unsigned long long t0 = g_now();
    for (uint32_t i = 1;; ++i) {
        if (g_try_wait(bar, parity)) return true;
        if ((i & 3u) == 0u && g_now() - t0 > kGemmWaitNs) return false;
    }
}

// g_wait by every lane of a warp, with a warp-uniform result.
__device__ __forceinline__ bool g_wait_warp(uint32_t bar, uint32_t parity) {
    return __all_sync(0xffffffffu, g_wait(bar, parity));
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

// 3-D tiled TMA load (no multicast) of box {x, y, z} into this CTA's shared memory.
__device__ __forceinline__ void g_tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                              uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

// `count` arrivals on `bar` at once.
__device__ __forceinline__ void g_arrive_n(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// 4-byte asynchronous copy global -> shared; `src_bytes` 0 fills zeros.
__device__ __forceinline__ void g_cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Arrive on `bar` once this thread's earlier cp.async copies have landed
// (the barrier's expected count includes this arrival).
__device__ __forceinline__ void g_cp_async_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
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

// The 4 MMAs (K = 16 each) of one stage, A from tensor memory (8 columns
// per K = 16 step), B from shared memory (32 bytes per step inside the
// swizzle atom), issued by one elected lane from a single asm block.
__device__ __forceinline__ void g_mma_stage_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_addr, uint32_t idesc,
                                               uint32_t accumulate) {
    // 32 bytes further inside the swizzle atom is +2 in the descriptor's
    // address field (addresses stay below 256 KB: no carry out of it)
    const uint64_t b0 = g_smem_desc(b_addr);
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %9, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %5, %10, p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %6, %10, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %7, %10, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %8, %10, 1;\n\t"
        "}\n" ::"r"(d_tmem),
        "r"(a_tmem), "r"(a_tmem + 8u), "r"(a_tmem + 16u), "r"(a_tmem + 24u), "l"(b0), "l"(b0 + 2u), "l"(b0 + 4u),
        "l"(b0 + 6u),
        "r"(accumulate), "r"(idesc)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued is done.
__device__ __forceinline__ void g_commit(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void g_tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void g_tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

__device__ __forceinline__ void g_tmem_ld16(uint32_t taddr, float (&f)[16]) {
    uint32_t v[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(v[i]);
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
// the final one to bf16.  int6 takes the two codes of a pair at p = 6 and
// p = 12 of one view of the code stream, int8 at p = 8, 4 and 12.
struct GDeq {
    uint64_t s_a, c_a;           // int6 (S6, S12) / int8 even pair (S8, S8), and -C_p * S_p
    uint64_t s_b, c_b;           // int8 odd pair (S4, S12)
};

__device__ __forceinline__ GDeq g_deq_consts(int qbits, float s) {
    auto sp = [&](int p) { return __fmul_rn(s, __int_as_float((127 - p) << 23)); };      // s * 2^-p
    auto cs = [&](int bits, int p) {                                                    // -C_p * S_p
        return __fmul_rn(-(8388608.0f + (float)(1 << (bits - 1 + p))), sp(p));
    };
    GDeq d;
    if (qbits == 6) {
        d.s_a = g_f2(sp(6), sp(12));
        d.c_a = g_f2(cs(6, 6), cs(6, 12));
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
// under the exponent of 2^23 (x = inverted bit | 0x4B000000, whose bits
// inside m are only the inverted one): (v & m) ^ x, one LOP3.
__device__ __forceinline__ float g_field(uint32_t v, uint32_t m, uint32_t x) {
    return __uint_as_float((v & m) ^ x);
}

__device__ __forceinline__ uint32_t g_pair_bf16(float f0, float f1, uint64_t s2, uint64_t c2) {
    uint64_t w2;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(w2) : "l"(g_f2(f0, f1)), "l"(s2), "l"(c2));
    float w0, w1;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(w0), "=f"(w1) : "l"(w2));
    return g_bf16x2(w0, w1);
}

// Codes 2i and 2i + 1 of a 64-code stage held in w[] (int6: 12 words and a
// zero; int8: 16 words) as one bf16x2 word of W_hat.
template <int QBITS>
__device__ __forceinline__ uint32_t g_pair(const uint32_t (&w)[16], int i, const GDeq& d) {
    if constexpr (QBITS == 6) {
        // the code stream shifted right by 12 i - 6 holds code 2i at bit 6
        // and code 2i + 1 at bit 12: one funnel shift per pair
        uint32_t v;
        if (i == 0) {
            v = w[0] << 6;
        } else {
            const int sh = 12 * i - 6;
            v = __funnelshift_r(w[sh >> 5], w[(sh >> 5) + 1], sh & 31);
        }
        return g_pair_bf16(g_field(v, 0xFC0u, 0x4B000800u), g_field(v, 0x3F000u, 0x4B020000u), d.s_a, d.c_a);
    } else {
        const uint32_t wd = w[i >> 1];
        if ((i & 1) == 0)                                  // bytes 0, 1: both at bit 8
            return g_pair_bf16(g_field(wd << 8, 0xFF00u, 0x4B008000u), g_field(wd, 0xFF00u, 0x4B008000u), d.s_a,
                               d.c_a);
        const uint32_t v = wd >> 12;                       // bytes 2, 3: at bits 4 and 12 of wd >> 12
        return g_pair_bf16(g_field(v, 0xFF0u, 0x4B000800u), g_field(v, 0xFF000u, 0x4B080000u), d.s_b, d.c_b);
    }
}

// One weight row's 64-code stage (at shared address `codes`) into the 32
// TMEM columns at `taddr` of this thread's lane.
template <int QBITS>
__device__ __forceinline__ void g_dequant_stage(uint32_t codes, uint32_t taddr, const GDeq& d) {
    uint32_t w[16];
    if constexpr (QBITS == 6) {
#pragma unroll
        for (int i = 0; i < 3; ++i)                        // 48 bytes, 16-byte aligned
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[4 * i]), "=r"(w[4 * i + 1]), "=r"(w[4 * i + 2]), "=r"(w[4 * i + 3])
                         : "r"(codes + 16u * i)
                         : "memory");
        w[12] = w[13] = w[14] = w[15] = 0u;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[4 * i]), "=r"(w[4 * i + 1]), "=r"(w[4 * i + 2]), "=r"(w[4 * i + 3])
                         : "r"(codes + 16u * i)
                         : "memory");
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t out[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) out[j] = g_pair<QBITS>(w, 16 * h + j, d);
        g_tmem_st16(taddr + 16u * (uint32_t)h, out);
    }
}

// Per-row constants of the fake-quant in the load.  The paired path below
// drops the clip to +-c and keeps only the clamp to +-qmax: for |w| <= c the
// clip does nothing, and for |w| > c both give +-qmax exactly when the
// row's own clip value lands there, RN(c / s) >= qmax (true for every
// binary32 scale and every normal binary16 one; a coarse binary16
// subnormal scale can break it).  Rows where this fails, or whose scale has
// no normal reciprocal, take the per-element path.
struct GFq {
    Scale S;
    bool paired;
};

__device__ __forceinline__ GFq g_fq_consts(const Scale& S) {
    GFq f;
    f.S = S;
    f.paired = false;
    if (S.fast && !S.zero) {
        const float t = __fdiv_rn(S.c, S.s);                       // < 256 for any scale make_scale gives
        const float q = __fsub_rn(__fadd_rn(t, kMagic), kMagic);   // round half to even
        f.paired = q >= S.qmaxf;
    }
    return f;
}

// The paired constants: (rcp, rcp), (kMagic, kMagic), (s, s).
struct GFq2 {
    uint64_t r2, m2, s2;
    float lo, hi;                // kMagic -+ qmax
};

// Two weights -> one bf16x2 word of W_hat on the paired path, and the larger
// distance of their scaled values from the rounded ones (the guard of the
// reciprocal quotient, as in the row kernel: at most 0.5 - 2^-13 means both
// codes are round_half_even(RN(w / s)), whether or not the code generator
// fuses the product into the sums; beyond it the caller redoes the weights
// with the exact division).  |w / s| >= 256 clamps to +-qmax on either side.
__device__ __forceinline__ uint32_t g_fq_pair(float w0, float w1, const GFq2& f, float& dmax) {
    uint64_t Y, B, N, E;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(Y) : "l"(g_f2(w0, w1)), "l"(f.r2));
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(B) : "l"(Y), "l"(f.m2));
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(N) : "l"(B), "l"(f.m2));
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(E) : "l"(Y), "l"(N));
    float e0, e1, b0, b1;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(e0), "=f"(e1) : "l"(E));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(b0), "=f"(b1) : "l"(B));
    dmax = fmaxf(dmax, fmaxf(fabsf(e0), fabsf(e1)));
    b0 = fminf(fmaxf(b0, f.lo), f.hi);
    b1 = fminf(fmaxf(b1, f.lo), f.hi);
    // w_hat = RN((b - kMagic) * s): the difference q is exact
    uint64_t Q, D;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(Q) : "l"(g_f2(b0, b1)), "l"(f.m2));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(Q), "l"(f.s2));
    float d0, d1;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(D));
    return g_bf16x2(d0, d1);
}

// One weight row's 64-wide stage, fake-quantized on the way into TMEM:
// w_hat = RN(q * s) with q = clamp(round_half_even(clip(w, -c, c) / s)), the
// very arithmetic of the fused row kernel (quantize_offset / offset_to_dq),
// then rounded to bf16 for the tensor cores.  The stage sits in shared
// memory as 128-byte rows with the 128-byte swizzle (16-byte chunk j of row r
// at chunk position j ^ (r & 7)): one row of 64 bf16, or two rows of 32 fp32
// in halves 16 KB apart.  Each group of 16 weights takes the paired path
// when the row allows it and redoes itself per element if its guard trips.
template <int DT>
__device__ __forceinline__ void g_fakequant_stage(uint32_t tile, int r, uint32_t taddr, const GFq& f) {
    const uint32_t sw = (uint32_t)(r & 7), row = tile + 128u * (uint32_t)r;
    auto fq = [&](float w) { return offset_to_dq(quantize_offset(w, f.S), f.S); };
    // 16-byte chunk c (0 .. 7) of the row's stage: 8 bf16 or 4 fp32 weights
    auto chunk = [&](int c, uint32_t (&u)[4]) {
        const uint32_t j = DT == kBF16 ? (uint32_t)c : (uint32_t)(c & 7);
        const uint32_t src = (DT == kBF16 ? row : row + (uint32_t)(c >> 3) * 128u * kGemmBN) + ((j ^ sw) << 4);
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3])
                     : "r"(src)
                     : "memory");
    };
    GFq2 f2;
    f2.r2 = g_f2(f.S.rcp, f.S.rcp);
    f2.m2 = g_f2(kMagic, kMagic);
    f2.s2 = g_f2(f.S.s, f.S.s);
    f2.lo = kMagic - f.S.qmaxf;
    f2.hi = kMagic + f.S.qmaxf;
    constexpr int kChunks = DT == kBF16 ? 2 : 4;           // chunks per 16 weights
#pragma unroll 1
    for (int g = 0; g < 4; ++g) {                          // 16 weights -> 8 bf16x2 columns
        uint32_t out[8];
        bool exact = !f.paired;
        if (f.paired) {
            float dmax = 0.0f;
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                uint32_t u[4];
                chunk(kChunks * g + c, u);
                if constexpr (DT == kBF16) {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        out[4 * c + e] = g_fq_pair(__uint_as_float(u[e] << 16), __uint_as_float(u[e] & 0xFFFF0000u),
                                                   f2, dmax);
                } else {
                    out[2 * c] = g_fq_pair(__uint_as_float(u[0]), __uint_as_float(u[1]), f2, dmax);
                    out[2 * c + 1] = g_fq_pair(__uint_as_float(u[2]), __uint_as_float(u[3]), f2, dmax);
                }
            }
            exact = dmax > kNearHalf;
        }
        if (exact) {
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                uint32_t u[4];
                chunk(kChunks * g + c, u);
                if constexpr (DT == kBF16) {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        out[4 * c + e] = g_bf16x2(fq(__uint_as_float(u[e] << 16)), fq(__uint_as_float(u[e] & 0xFFFF0000u)));
                } else {
                    out[2 * c] = g_bf16x2(fq(__uint_as_float(u[0])), fq(__uint_as_float(u[1])));
                    out[2 * c + 1] = g_bf16x2(fq(__uint_as_float(u[2])), fq(__uint_as_float(u[3])));
                }
            }
        }
        g_tmem_st8(taddr + 8u * (uint32_t)g, out);
    }
}

// -------------------------------------------------------- chunk schedule --

// The block's chunks in order, walked incrementally (no division in the
// loops: a 64-bit division costs far more than a hand-off).  The block owns
// the stage units [u0, u1) (stream-K, tile-major) or whole tiles blockIdx.x,
// blockIdx.x + gridDim.x, ...; a chunk is the part of one aligned run of CS
// K stages of one tile that the block owns: sub-stages lo .. hi.  A segment
// is a run of the block's chunks of one tile.
struct CIter {
    int64_t tile, step;
    int64_t rem;                 // stages of the block not yet walked
    int64_t seq;                 // chunk index within the block
    int kt, KT, CS;
    int c, lo, hi;               // the chunk: index within the tile, first and last owned sub-stage
    bool seg_first, seg_last, seg_full;
    int seg_kt0;
    __device__ __forceinline__ void set() {
        c = kt / CS;                                       // 32-bit: cheap
        lo = kt - c * CS;
        const int chunk_end = min(CS - 1, KT - 1 - c * CS);
        hi = (int)min((int64_t)chunk_end, (int64_t)lo + rem - 1);
        seg_first = kt == 0 || seq == 0;
        if (seg_first) seg_kt0 = kt;
        const int kt_last = c * CS + hi;
        seg_last = kt_last == KT - 1 || rem == (int64_t)(hi - lo + 1);
        seg_full = seg_kt0 == 0 && kt_last == KT - 1;
    }
    __device__ __forceinline__ void init(const GemmParams& P) {
        KT = P.kt_per_tile;
        CS = P.cs;
        seq = 0;
        if (P.streamk) {
            const int64_t total = P.tiles * (int64_t)KT;
            const int64_t u0 = total * (int64_t)blockIdx.x / gridDim.x;
            const int64_t u1 = total * ((int64_t)blockIdx.x + 1) / gridDim.x;
            rem = u1 - u0;
            tile = u0 / KT;
            kt = (int)(u0 - tile * KT);
            step = 1;
        } else {
            const int64_t my = P.tiles > (int64_t)blockIdx.x ? (P.tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
            rem = my * KT;
            tile = blockIdx.x;
            kt = 0;
            step = gridDim.x;
        }
        seg_kt0 = kt;
        if (rem > 0) set();
    }
    __device__ __forceinline__ bool valid() const { return rem > 0; }
    __device__ __forceinline__ void next() {
        const int n = hi - lo + 1;
        rem -= n;
        kt += n;
        if (kt == KT) {
            kt = 0;
            tile += step;
        }
        ++seq;
        if (rem > 0) set();
    }
};

// Slot and phase of a ring of D barriers or buffers, advanced one use at a time.
struct GRing {
    int s, D;
    uint32_t ph;
    __device__ __forceinline__ void init(int depth) {
        s = 0;
        D = depth;
        ph = 0u;
    }
    __device__ __forceinline__ void next() {
        if (++s == D) {
            s = 0;
            ph ^= 1u;
        }
    }
};

// ----------------------------------------------------------------- kernel --

// WM: 0 = packed codes (dequant on load), 1 = bf16 / fp32 weights and clips
// (fake-quant on load); two instantiations, so that neither pays the
// other's registers.
template <int WM>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_dequant_kernel(const __grid_constant__ GemmParams P) {
    extern __shared__ unsigned char g_smem[];
    const uint32_t raw = g_smem_u32(g_smem);
    const uint32_t base = (raw + 1023u) & ~1023u;          // SWIZZLE_128B tiles: 1024-byte aligned
    const int DX = P.dx, DC = P.dc, DW = P.dw, DD = P.dd, NT = P.nt, NI = P.ni, CS = P.cs;
    const int XS = P.xs, XPC = CS / XS;                    // stages per X slot, X slots per chunk
    const uint32_t xs_bytes = (uint32_t)NT * 128u;         // one stage of X
    const uint32_t x_bytes = xs_bytes * (uint32_t)XS;      // an X slot
    // bytes of a row's 64-wide stage in a code slot: packed codes, or the
    // weights themselves in the weight modes (bf16: one 128-byte swizzled
    // row; fp32: two 128-byte halves, 16 KB apart)
    const uint32_t cb = P.wmode == 1 ? 128u : P.wmode == 2 ? 256u : P.qbits == 6 ? 48u : 64u;
    const uint32_t crow = cb * (uint32_t)CS;               // bytes of a row's chunk
    const uint32_t c_bytes = (uint32_t)kGemmBN * crow;     // a code chunk slot
    // [X ring][code ring][barriers]
    const uint32_t cs0 = base + (uint32_t)DX * x_bytes;
    const uint32_t bars = base + (uint32_t)(kGemmSmemBytes - 1024 - kGemmBarBytes);
    auto full_x = [&](int s) { return bars + 8u * (uint32_t)s; };
    auto x_done = [&](int s) { return bars + 8u * (uint32_t)(kGemmMaxX + s); };   // an X slot's MMAs are done
    constexpr int kB0 = 2 * kGemmMaxX;
    auto full_c = [&](int s) { return bars + 8u * (uint32_t)(kB0 + s); };
    auto empty_c = [&](int s) { return bars + 8u * (uint32_t)(kB0 + kGemmMaxC + s); };
    auto full_w = [&](int s, int k) {                      // sub-stage k of W_hat chunk slot s
        return bars + 8u * (uint32_t)(kB0 + 2 * kGemmMaxC + s * CS + k);
    };
    auto done = [&](int s) {                               // a chunk's MMA commit (frees its W_hat slot)
        return bars + 8u * (uint32_t)(kB0 + 2 * kGemmMaxC + kGemmMaxWS + s);
    };
    const uint32_t acc_full0 =
        bars + 8u * (uint32_t)(kB0 + 2 * kGemmMaxC + kGemmMaxWS + kGemmMaxDone);
    auto acc_full = [&](int j) { return acc_full0 + 8u * (uint32_t)j; };   // issuer j's segment sums are ready
    const uint32_t acc_empty = acc_full0 + 16u;                             // the epilogue has read them
    const uint32_t fin = acc_full0 + 24u;                                   // 2 barriers: an issuer's MMAs are all done
    const uint32_t tmem_slot = acc_full0 + 40u;
    auto x_tile = [&](int s) { return base + (uint32_t)s * x_bytes; };
    auto c_tile = [&](int s) { return cs0 + (uint32_t)s * c_bytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    CIter it;
    it.init(P);

    if (threadIdx.x == 0) {
        for (int s = 0; s < DX; ++s) {
            g_bar_init(full_x(s), 1);
            g_bar_init(x_done(s), 1);
        }
        for (int s = 0; s < DC; ++s) {
            g_bar_init(full_c(s), P.code_copy ? 32 : 1);
            g_bar_init(empty_c(s), 4 * CS);                // four warps per sub-stage
        }
        for (int s = 0; s < DW; ++s)
            for (int k = 0; k < CS; ++k) g_bar_init(full_w(s, k), 4);
        for (int s = 0; s < DD; ++s) g_bar_init(done(s), 1);
        g_bar_init(acc_full(0), 1);
        g_bar_init(acc_full(1), 1);
        g_bar_init(acc_empty, 4);                          // the four epilogue warps
        g_bar_init(fin, 1);
        g_bar_init(fin + 8u, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (!P.code_copy)
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tmap_w)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tmap_x)) : "memory");
    }
    if (warp == 3) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(tmem_slot)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    uint32_t tmem;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(tmem) : "r"(tmem_slot) : "memory");
    const uint32_t w_col0 = (uint32_t)NI * P.acc_cols;     // W_hat chunk slots after the accumulators

    bool ok = true;
    if (warp == 0) {
        // ------------------------------------------------ code producer --
        GRing rc;
        rc.init(DC);
        int64_t cur_tile = -1;
        int n0 = 0;
        int64_t issued = 0;
        for (; it.valid() && ok; it.next(), rc.next()) {
            if (it.tile != cur_tile) {
                cur_tile = it.tile;
                n0 = (int)(it.tile / P.tiles_m) * kGemmBN;
            }
            // the slot's previous chunk has been read by its dequant warps
            if (it.seq >= DC && !g_wait_warp(empty_c(rc.s), rc.ph ^ 1u)) {
                ok = false;
                break;
            }
            if (WM != 0) {
                // weight modes (one stage per chunk): the stage's 128 x 64
                // weights, 128-byte swizzled rows; K past the end zero-filled
                if (lane == 0) {
                    g_arrive_tx(full_c(rc.s), c_bytes);
                    const int kx = it.c * kGemmBK;
                    if (P.wmode == 1) {
                        g_tma_load_2d(c_tile(rc.s), &P.tmap_w, kx, n0, full_c(rc.s));
                    } else if (P.w3d) {
                        g_tma_load_3d(c_tile(rc.s), &P.tmap_w, 0, n0, 2 * it.c, full_c(rc.s));
                    } else {
                        g_tma_load_2d(c_tile(rc.s), &P.tmap_w, kx, n0, full_c(rc.s));
                        g_tma_load_2d(c_tile(rc.s) + 128u * kGemmBN, &P.tmap_w, kx + 32, n0, full_c(rc.s));
                    }
                }
            } else if (!P.code_copy) {
                if (lane == 0) {
                    g_arrive_tx(full_c(rc.s), c_bytes);    // out-of-range rows / bytes are zero-filled
                    g_tma_load_2d(c_tile(rc.s), &P.tmap_w, it.c * (int)crow, n0, full_c(rc.s));
                }
            } else {
                // 4-byte copies of every row's chunk bytes; past the row end
                // and past the last weight row zeros are filled in
                const uint32_t words = crow / 4u;
                const int64_t off0 = (int64_t)it.c * crow;
                for (uint32_t e = (uint32_t)lane; e < (uint32_t)kGemmBN * words; e += 32u) {
                    const uint32_t r = e / words, wi = e - r * words;
                    const int64_t n = n0 + r;
                    const int64_t off = off0 + 4 * wi;
                    const bool in = n < P.N && off + 4 <= P.prb;
                    const uint8_t* src = in ? P.codes + n * P.prb + off : P.codes;
                    g_cp_async4(c_tile(rc.s) + r * crow + 4u * wi, src, in ? 4u : 0u);
                }
                g_cp_async_arrive(full_c(rc.s));
            }
            // sub-stages the block does not own are released here, so that the
            // slot's release count is always four warps per sub-stage
            const int missing = CS - (it.hi - it.lo + 1);
            if (lane == 0 && missing > 0) g_arrive_n(empty_c(rc.s), 4u * (uint32_t)missing);
            issued = it.seq + 1;
        }
        // no copy may still be landing when the block exits
        for (int64_t q = max((int64_t)0, issued - DC); q < issued; ++q)
            if (!g_wait_warp(full_c((int)(q % DC)), (uint32_t)((q / DC) & 1))) ok = false;
    } else if (warp == 3) {
        // --------------------------------------------------- X producer --
        GRing rx;                                          // X slots
        rx.init(DX);
        int64_t cur_tile = -1;
        int m0 = 0;
        int64_t xseq = 0;                                  // X slots issued
        for (; it.valid() && ok; it.next()) {
            if (it.tile != cur_tile) {
                cur_tile = it.tile;
                m0 = (int)(it.tile % P.tiles_m) * NT;
            }
            for (int j = 0; j < XPC && ok; ++j, rx.next(), ++xseq) {
                // the slot's previous stages have been consumed by their MMAs
                if (xseq >= DX && !g_wait_warp(x_done(rx.s), rx.ph ^ 1u)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const int k0 = j * XS;
                    if (P.x3d) {
                        g_arrive_tx(full_x(rx.s), x_bytes);    // K stages past the end are zero-filled
                        g_tma_load_3d(x_tile(rx.s), &P.tmap_x, 0, m0, it.c * CS + k0, full_x(rx.s));
                    } else {
                        const int a = max(k0, it.lo), b = min(k0 + XS - 1, it.hi);
                        g_arrive_tx(full_x(rx.s), b >= a ? xs_bytes * (uint32_t)(b - a + 1) : 0u);
                        for (int k = a; k <= b; ++k)
                            g_tma_load_2d(x_tile(rx.s) + (uint32_t)(k - k0) * xs_bytes, &P.tmap_x,
                                          (it.c * CS + k) * kGemmBK, m0, full_x(rx.s));
                    }
                }
            }
        }
        for (int64_t q = max((int64_t)0, xseq - DX); q < xseq; ++q)
            if (!g_wait_warp(full_x((int)(q % DX)), (uint32_t)((q / DX) & 1))) ok = false;
    } else if (warp == 1 || warp == 2) {
        // -------------------------------------------------------- MMA --
        const int j = warp - 1;
        if (j < NI) {
            const uint32_t acc = tmem + (uint32_t)j * P.acc_cols;
            GRing rx, rw, rd;                              // X slot, W_hat slot, commit of the chunk
            rx.init(DX);
            rw.init(DW);
            rd.init(DD);
            uint32_t seg_ph = 0u;                          // parity of the epilogue's next acc_empty phase
            bool fresh = true;                             // next MMA into acc starts a sum
            int mine = 0;                                  // seq % NI, kept incrementally
            for (; it.valid() && ok; it.next(), rw.next(), rd.next(), mine = mine + 1 == NI ? 0 : mine + 1) {
                if (it.seg_first && it.seq > 0) {
                    // a new segment: the epilogue must have read the previous one
                    if (!g_wait_warp(acc_empty, seg_ph)) ok = false;
                    seg_ph ^= 1u;
                    fresh = true;
                }
                if (!ok) break;
                if (mine != j) {                           // the other issuer's chunk: keep the X ring in step
                    for (int xj = 0; xj < XPC; ++xj) rx.next();
                } else {
                    for (int xj = 0; xj < XPC && ok; ++xj, rx.next()) {
                        const int k0 = xj * XS, a = max(k0, it.lo), b = min(k0 + XS - 1, it.hi);
                        // waited even without a stage to run: the slot may be
                        // refilled only after this copy has landed
                        if (!g_wait_warp(full_x(rx.s), rx.ph)) {
                            ok = false;
                            break;
                        }
                        for (int k = a; k <= b; ++k) {
                            if (!g_wait_warp(full_w(rw.s, k), rw.ph)) {
                                ok = false;
                                break;
                            }
                            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                            g_mma_stage_ts(acc, tmem + w_col0 + 32u * (uint32_t)(rw.s * CS + k),
                                           x_tile(rx.s) + (uint32_t)(k - k0) * xs_bytes, P.idesc, fresh ? 0u : 1u);
                            fresh = false;
                        }
                        if (!ok) break;
                        g_commit(x_done(rx.s));            // the X slot is free once these MMAs are done
                    }
                    if (!ok) break;
                    g_commit(done(rd.s));                  // the chunk's W_hat slot likewise
                }
                if (it.seg_last) g_commit(acc_full(j));    // the segment's sums (of this issuer) are complete
            }
            g_commit(fin + 8u * (uint32_t)j);
            if (!g_wait_warp(fin + 8u * (uint32_t)j, 0u)) ok = false;
        }
    } else if (warp >= kGemmEpi0 && warp < kGemmEpi0 + 4) {
        // --------------------------------------------------- epilogue --
        const int quarter = warp & 3;
        uint32_t par = 0u;
        int64_t seg_seq0 = 0;
        for (; it.valid() && ok; it.next()) {
            if (it.seg_first) seg_seq0 = it.seq;
            if (!it.seg_last) continue;
            // issuers holding a partial sum of this segment
            const int64_t len = it.seq - seg_seq0 + 1;
            const int nacc = (int)min((int64_t)NI, len);
            for (int a = 0; a < NI; ++a)
                if (!g_wait_warp(acc_full(a), par)) ok = false;
            par ^= 1u;
            if (!ok) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const int64_t n = (it.tile / P.tiles_m) * kGemmBN + 32 * quarter + lane;
            const int64_t m0 = (it.tile % P.tiles_m) * NT;
            const int first_acc = (int)(seg_seq0 % NI);
            const bool full = it.seg_full;
            for (int c = 0; c < NT; c += 16) {
                float v[16];
                g_tmem_ld16(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)first_acc * P.acc_cols + (uint32_t)c,
                            v);
                if (nacc == 2) {
                    float v2[16];
                    g_tmem_ld16(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(1 - first_acc) * P.acc_cols +
                                    (uint32_t)c,
                                v2);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = __fadd_rn(v[i], v2[i]);
                }
                if (n < P.N) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int64_t m = m0 + c + i;
                        if (m < P.M) {
                            float* dst = P.y + m * P.ldy + n;   // a warp writes 32 consecutive floats
                            if (full) *dst = v[i];
                            else atomicAdd(dst, v[i]);
                        }
                    }
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) g_arrive(acc_empty);
        }
    } else if (warp >= kGemmDq0) {
        // ---------------------------------------------------- dequant --
        const int grp = (warp - kGemmDq0) >> 2, quarter = warp & 3;
        const int r = 32 * quarter + lane;                 // weight row of the tile, TMEM lane
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * quarter) << 16) + w_col0;
        GRing rc, rw, rd;                                  // code slot, W_hat slot, commit of chunk seq - DW
        rc.init(DC);
        rw.init(DW);
        rd.init(DD);
        // group grp takes sub-stage grp % CS of the chunks with seq % (4 / CS) == grp / CS
        const int cpg = kGemmGroups / CS, my_pc = grp / CS, k = grp % CS;
        int pc = 0;                                        // seq % cpg, kept incrementally
        int64_t cur_tile = -1;
        GDeq deq{};
        GFq fq{};                                          // weight modes: the row's clip and scale
        for (; it.valid() && ok; it.next(), rc.next(), rw.next(), pc = pc + 1 == cpg ? 0 : pc + 1) {
            const bool reuse = it.seq >= DW;
            const int rd_s = rd.s;
            const uint32_t rd_ph = rd.ph;
            if (reuse) rd.next();                          // now at chunk seq - DW + 1
            if (pc != my_pc) continue;
            // the W_hat slot is free once the commit of chunk seq - DW is in
            if (reuse && !g_wait_warp(done(rd_s), rd_ph)) {
                ok = false;
                break;
            }
            if (k < it.lo || k > it.hi) {
                // a sub-stage the block does not own: nothing to dequantize,
                // but its W_hat barrier still completes a phase (keeping the
                // slot's phases in step); the code slot's release for it was
                // counted by the code producer
                __syncwarp();
                if (lane == 0) g_arrive(full_w(rw.s, k));
                continue;
            }
            if (it.tile != cur_tile) {
                cur_tile = it.tile;
                const int64_t n = (it.tile / P.tiles_m) * kGemmBN + r;
                if constexpr (WM == 0) {
                    const float srow = n < P.N ? __half2float(__ushort_as_half(P.scale[n])) : 0.0f;
                    deq = g_deq_consts(P.qbits, srow);
                } else {
                    uint16_t hb;
                    bool range;
                    const float c = n < P.N ? P.clip[n] : 0.0f;
                    fq = g_fq_consts(make_scale(__float_as_uint(c), P.qbits == 6 ? 31 : 127, P.export_scale != 0,
                                                &hb, &range));
                    if (range && P.status) atomicOr(reinterpret_cast<unsigned int*>(P.status), 0x2u);
                }
            }
            if (!g_wait_warp(full_c(rc.s), rc.ph)) {
                ok = false;
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t codes = c_tile(rc.s) + (uint32_t)r * crow + (uint32_t)k * cb;
            const uint32_t taddr = lane_addr + 32u * (uint32_t)(rw.s * CS + k);
            if constexpr (WM != 0) {
                if (P.wmode == 1) g_fakequant_stage<kBF16>(c_tile(rc.s), r, taddr, fq);
                else g_fakequant_stage<kF32>(c_tile(rc.s), r, taddr, fq);
            } else {
                if (P.qbits == 6) g_dequant_stage<6>(codes, taddr, deq);
                else g_dequant_stage<8>(codes, taddr, deq);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                g_arrive(empty_c(rc.s));                   // every lane's code loads have been used
                g_arrive(full_w(rw.s, k));
            }
        }
    }
    if (!ok && lane == 0 && P.status) atomicOr(reinterpret_cast<unsigned int*>(P.status), 0x4u);
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 3) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

}  // namespace gq
