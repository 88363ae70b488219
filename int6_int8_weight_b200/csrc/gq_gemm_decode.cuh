// gq_gemm_decode.cuh -- the dequant-on-load GEMM for decode-sized batches
// (M <= 16 tokens): Y[M, N] = X[M, K] * W_hat[N, K]^T with the same W_hat
// as gq_gemm.cuh (bf16(RN(q * s)) from the packed codes and binary16 row
// scales of an export), computed with register-level tensor-core MMAs.
//
// Why a second kernel.  With 16 tokens the contraction is bound by the code
// stream (2 FLOP per code per token): the tensor pipe of the tcgen05 kernel
// is a few percent busy, and its cost is the pipeline around it (a code
// producer, MMA issuers and dequant warps handing stages to one another
// through mbarriers and tensor memory).  Here every warp streams its own 16
// weight rows into a shared-memory ring of its own (one TMA box of 16 rows x
// one super-stage of packed bytes per copy, kDecD super-stages deep, so that
// enough bytes are in flight to cover the memory latency), dequantizes them
// into the B fragments of mma.sync.m16n8k16 (bf16 in, fp32 accumulate), and
// no warp waits on another except at the block's unit boundaries.
//
// K permutation.  A sum over k is unchanged when X and W_hat are permuted
// alike along k.  Within every 256-wide super-stage, lane t (t = lane % 4)
// of a quad feeds the MMA's k positions {2t, 2t+1, 2t+8, 2t+9} of k-block b
// (b = 0..15) with the physical pairs 32t + 2b and 32t + 2b + 1 (pair p =
// k elements 2p, 2p+1).  Lane t thus owns the physical k range
// [64t, 64t + 64) of the super-stage: for int6 the 48 contiguous bytes at
// 48t (4 codes per 3 bytes), for int8 the 64 bytes at 64t, and 128 bytes of
// X rows g and g + 8.  The packed rows must suit TMA (a pitch that is a
// multiple of 16 bytes); other shapes go to the tcgen05 kernel.
//
// Work: units of 256 weight rows (16 warps x 16 rows; a warp owns two
// 8-row MMA column groups) x 512 of K (two super-stages), N-major; each
// block takes a contiguous run of units, keeps its accumulators across the
// units of one row block and adds them into Y (zeroed by the host) when the
// row block changes.  The X slice of a unit (16 x 512 bf16, zero-filled
// past M and K) is staged in shared memory by cp.async, double-buffered
// across units (issued at the start of the unit before, waited at its own
// start), its 16-byte chunks XOR-swizzled so that the lanes of a quad read
// different banks.  TMA zero-fills codes past the end of a row or past the
// last weight row.  Every wait on a ring barrier is bounded; an expired
// wait sets GQ_STATUS_TIMEOUT, and the warp stops issuing and computing but
// keeps the block's barriers and, before it exits, waits (bounded) for its
// copies in flight.
#pragma once

#include "gq_gemm.cuh"

namespace gq {

constexpr int kDecWarps = 16;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecNG = 2;                                // 8-row column groups per warp
constexpr int kDecRows = kDecWarps * 8 * kDecNG;         // 256 weight rows per unit
constexpr int kDecSS = 256;                              // K per super-stage
constexpr int kDecKc = 2 * kDecSS;                       // K per unit
constexpr int kDecPitch = kDecKc + 32;                   // X slice row pitch (bf16): 64-byte pad
constexpr int kDecD = 3;                                 // code ring depth (super-stages)
constexpr int64_t kDecMaxM = 16;                         // batches up to one MMA row tile
constexpr int kDecXBytes = 2 * 16 * kDecPitch * 2;       // two X slices
constexpr unsigned long long kDecWaitNs = 4000000000ull;
template <int QBITS>
__host__ __device__ constexpr int dec_ss_bytes() { return QBITS == 6 ? 192 : 256; }   // a row's super-stage
template <int QBITS>
__host__ __device__ constexpr int dec_ring_bytes() { return kDecWarps * kDecD * 16 * dec_ss_bytes<QBITS>(); }
template <int QBITS>
__host__ __device__ constexpr int dec_smem_bytes() {
    return 128 /* alignment */ + kDecXBytes + dec_ring_bytes<QBITS>() + kDecWarps * kDecD * 8;
}
static_assert(dec_smem_bytes<8>() <= 232448, "decode kernel shared memory");

struct DecParams {
    CUtensorMap tmap;           // codes [N, prb] bytes, box {super-stage bytes, 16 rows}, no swizzle
    const uint16_t* x;          // [M, ldx] bf16
    const uint16_t* scale;      // [N] binary16
    float* y;                   // [M, ldy] fp32, zeroed
    int32_t* status;            // nullable: GQ_STATUS_TIMEOUT on an expired wait
    int64_t ldx, ldy, M, N, K;
    int64_t units, kunits;      // units = row blocks * kunits
};

__device__ __forceinline__ void dec_cp_async16(uint32_t dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void dec_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Per-row dequant constants as scalars (the same identity as GDeq:
// q * s = F * S_p - C_p * S_p, one fused multiply-add per code), for
// scalar fused multiply-adds on the FMA pipe: the decode kernel is bound by
// the integer pipe, which the register-pair moves of the paired form use.
struct DecDeq {
    float s0, c0, s1, c1;        // int6: p = 6, 12; int8 even pair: p = 8, 8
    float s2, c2, s3, c3;        // int8 odd pair: p = 4, 12
};

__device__ __forceinline__ DecDeq dec_deq_consts(int qbits, float s) {
    auto sp = [&](int p) { return __fmul_rn(s, __int_as_float((127 - p) << 23)); };      // s * 2^-p
    auto cs = [&](int bits, int p) {                                                    // -C_p * S_p
        return __fmul_rn(-(8388608.0f + (float)(1 << (bits - 1 + p))), sp(p));
    };
    DecDeq d;
    if (qbits == 6) {
        d.s0 = sp(6); d.c0 = cs(6, 6); d.s1 = sp(12); d.c1 = cs(6, 12);
        d.s2 = d.c2 = d.s3 = d.c3 = 0.0f;
    } else {
        d.s0 = d.s1 = sp(8); d.c0 = d.c1 = cs(8, 8);
        d.s2 = sp(4); d.c2 = cs(8, 4); d.s3 = sp(12); d.c3 = cs(8, 12);
    }
    return d;
}

// Codes 2i and 2i + 1 of the lane's window w[] (int6: pair i at bit 12 i;
// int8: bytes 2i, 2i + 1) as one bf16x2 word of W_hat; the fields are those
// of g_pair.
template <int QBITS>
__device__ __forceinline__ uint32_t dec_pair(const uint32_t (&w)[16], int i, const DecDeq& d) {
    if constexpr (QBITS == 6) {
        uint32_t v;
        if (i == 0) {
            v = w[0] << 6;
        } else {
            const int sh = 12 * i - 6;
            v = __funnelshift_r(w[sh >> 5], w[(sh >> 5) + 1], sh & 31);
        }
        return g_bf16x2(__fmaf_rn(g_field(v, 0xFC0u, 0x4B000800u), d.s0, d.c0),
                        __fmaf_rn(g_field(v, 0x3F000u, 0x4B020000u), d.s1, d.c1));
    } else {
        const uint32_t wd = w[i >> 1];
        if ((i & 1) == 0)
            return g_bf16x2(__fmaf_rn(g_field(wd << 8, 0xFF00u, 0x4B008000u), d.s0, d.c0),
                            __fmaf_rn(g_field(wd, 0xFF00u, 0x4B008000u), d.s1, d.c1));
        const uint32_t v = wd >> 12;
        return g_bf16x2(__fmaf_rn(g_field(v, 0xFF0u, 0x4B000800u), d.s2, d.c2),
                        __fmaf_rn(g_field(v, 0xFF000u, 0x4B080000u), d.s3, d.c3));
    }
}

// Byte offset of 16-byte chunk c (0 .. 63) of X slice row m: chunk c sits
// at position c ^ ((c >> 3) & 7), so that the four lanes of a quad, which
// read chunks 32 ss + 8 t + i at the same time, hit different banks (and
// rows g and g + 1, 64 bytes apart mod 128, do too).
__device__ __forceinline__ uint32_t dec_x_off(int m, int c) {
    return (uint32_t)(m * kDecPitch) * 2u + 16u * (uint32_t)(c ^ ((c >> 3) & 7));
}

// This thread's share of X[:, k0 .. k0 + 512) into the slice buffer at `dst`:
// 16-byte cp.async copies, zero-filled past M and K.  Not committed here.
__device__ __forceinline__ void dec_load_x(const DecParams& P, uint32_t dst, int64_t k0) {
    for (int e = threadIdx.x; e < 16 * (kDecKc / 8); e += kDecThreads) {
        const int m = e / (kDecKc / 8), c = e % (kDecKc / 8);
        const int64_t k = k0 + 8 * c;
        int64_t n = (m < P.M) ? min((int64_t)8, P.K - k) : 0;
        if (n < 0) n = 0;
        const uint16_t* src = n > 0 ? P.x + m * P.ldx + k : P.x;
        dec_cp_async16(dst + dec_x_off(m, c), src, (uint32_t)n * 2u);
    }
}

template <int QBITS>
__global__ void __launch_bounds__(kDecThreads, 1) gemm_decode_kernel(const __grid_constant__ DecParams P) {
    constexpr int SSB = dec_ss_bytes<QBITS>();            // packed bytes of a row's super-stage
    constexpr int LC = SSB / 64;                           // a lane's 16-byte chunks of a row (3 or 4)
    constexpr uint32_t kBox = 16u * SSB;                   // one ring slot: the warp's 16 rows
    extern __shared__ __align__(128) unsigned char dec_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int64_t G = gridDim.x;
    const int64_t u0 = P.units * (int64_t)blockIdx.x / G, u1 = P.units * ((int64_t)blockIdx.x + 1) / G;
    if (u0 >= u1) return;
    const uint32_t xs0 = (static_cast<uint32_t>(__cvta_generic_to_shared(dec_smem)) + 127u) & ~127u;
    const uint32_t xbuf_bytes = 16u * kDecPitch * 2u;
    const uint32_t ring = xs0 + kDecXBytes + (uint32_t)warp * (kDecD * kBox);
    const uint32_t bars = xs0 + kDecXBytes + kDecWarps * kDecD * kBox + (uint32_t)warp * (kDecD * 8);
    if (lane == 0) {
        for (int d = 0; d < kDecD; ++d) g_bar_init(bars + 8u * (uint32_t)d, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tmap)) : "memory");
    }
    __syncwarp();
    const int64_t T = (u1 - u0) * 2;                       // super-stages of the block
    const int64_t row_lane = (int64_t)warp * (8 * kDecNG) + g;   // + 8 j: the lane's B column rows
    bool ok = true;

    // ---- issue side: (row block, K unit, super-stage), walked incrementally
    int64_t is_nb = u0 / P.kunits, is_kb = u0 - (u0 / P.kunits) * P.kunits;
    int is_ss = 0;
    int64_t issued = 0;
    auto issue = [&]() {
        if (issued >= T || !ok) return;
        if (lane == 0) {
            const uint32_t d = (uint32_t)(issued % kDecD);
            g_arrive_tx(bars + 8u * d, kBox);              // rows past N and bytes past the row are zero-filled
            g_tma_load_2d(ring + d * kBox, &P.tmap, (int)((is_kb * 2 + is_ss) * SSB),
                          (int)(is_nb * kDecRows + warp * 16), bars + 8u * d);
        }
        ++issued;
        if (++is_ss == 2) {
            is_ss = 0;
            if (++is_kb == P.kunits) {
                is_kb = 0;
                ++is_nb;
            }
        }
    };

    // ---- compute side
    int64_t cp_nb = u0 / P.kunits, cp_kb = u0 - cp_nb * P.kunits;
    float acc[kDecNG][4];
    DecDeq deq[kDecNG];
    int64_t cur_nb = -1;
    auto flush = [&]() {
        // lane holds Y[g][n], Y[g][n + 1], Y[g + 8][n], Y[g + 8][n + 1], n = row block + 8 j + 2 t
#pragma unroll
        for (int j = 0; j < kDecNG; ++j) {
            const int64_t n = cur_nb * kDecRows + (int64_t)warp * (8 * kDecNG) + 8 * j + 2 * t;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t m = g + 8 * h;
                if (m < P.M) {
                    if (n < P.N) atomicAdd(P.y + m * P.ldy + n, acc[j][2 * h]);
                    if (n + 1 < P.N) atomicAdd(P.y + m * P.ldy + n + 1, acc[j][2 * h + 1]);
                }
            }
        }
    };

    dec_load_x(P, xs0, cp_kb * kDecKc);
    asm volatile("cp.async.commit_group;" ::: "memory");
    for (int d = 0; d < kDecD; ++d) issue();               // the first kDecD super-stages in flight
    int64_t waited = 0;
    for (int64_t tt = 0; tt < T; ++tt) {
        const int ss = (int)(tt & 1);
        const int64_t ui = tt >> 1;                        // unit index within the block
        if (ss == 0) {
            // a new unit: every thread's share of its X slice has landed, and
            // every warp is done with the previous unit, whose X buffer the
            // next unit's slice takes
            if (ui > 0 && ++cp_kb == P.kunits) {
                cp_kb = 0;
                ++cp_nb;
            }
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            __syncthreads();
            if (u0 + ui + 1 < u1) {
                dec_load_x(P, xs0 + (uint32_t)((ui + 1) & 1) * xbuf_bytes,
                           (cp_kb + 1 == P.kunits ? 0 : cp_kb + 1) * kDecKc);
                asm volatile("cp.async.commit_group;" ::: "memory");
            }
            if (cp_nb != cur_nb) {
                if (cur_nb >= 0 && ok) flush();
                cur_nb = cp_nb;
#pragma unroll
                for (int j = 0; j < kDecNG; ++j) {
                    acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
                    const int64_t n = cp_nb * kDecRows + row_lane + 8 * j;
                    const float srow = n < P.N ? __half2float(__ushort_as_half(P.scale[n])) : 0.0f;
                    deq[j] = dec_deq_consts(QBITS, srow);
                }
            }
        }
        const int d = (int)(tt % kDecD);
        if (ok) {
            if (g_wait_warp(bars + 8u * (uint32_t)d, (uint32_t)((tt / kDecD) & 1))) {
                ++waited;
            } else {
                ok = false;
                if (lane == 0 && P.status) atomicOr(reinterpret_cast<unsigned int*>(P.status), 0x4u);
            }
        }
        if (ok) {
            const uint32_t xb = xs0 + (uint32_t)(ui & 1) * xbuf_bytes;
            // the lane's code words of its two rows (row 8 j + g of the slot)
            uint32_t cw[kDecNG][16];
#pragma unroll
            for (int j = 0; j < kDecNG; ++j) {
                const uint32_t src = ring + (uint32_t)d * kBox + (uint32_t)((8 * j + g) * SSB + (SSB / 4) * t);
#pragma unroll
                for (int c = 0; c < LC; ++c)
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(cw[j][4 * c]), "=r"(cw[j][4 * c + 1]), "=r"(cw[j][4 * c + 2]),
                                   "=r"(cw[j][4 * c + 3])
                                 : "r"(src + 16u * (uint32_t)c));
#pragma unroll
                for (int w = 4 * LC; w < 16; ++w) cw[j][w] = 0u;
            }
            // X rows g and g + 8 of this super-stage: chunk 32 ss + 8 t + q sits at
            // 32 ss + 8 t + (q ^ r), r = (4 ss + t) & 7 (dec_x_off)
            const uint32_t xg = xb + (uint32_t)(g * kDecPitch) * 2u + 16u * (uint32_t)(32 * ss + 8 * t);
            const uint32_t r = (uint32_t)((4 * ss + t) & 7);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                // physical pairs 32 t + 8 s .. + 7: chunks q = 2 s, 2 s + 1 of the lane's eight
                uint32_t xa[8], xc[8];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t a = xg + 16u * (((uint32_t)(2 * s + h)) ^ r);
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(xa[4 * h]), "=r"(xa[4 * h + 1]), "=r"(xa[4 * h + 2]), "=r"(xa[4 * h + 3])
                                 : "r"(a));
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(xc[4 * h]), "=r"(xc[4 * h + 1]), "=r"(xc[4 * h + 2]), "=r"(xc[4 * h + 3])
                                 : "r"(a + (uint32_t)(8 * kDecPitch) * 2u));
                }
#pragma unroll
                for (int j = 0; j < kDecNG; ++j) {
                    uint32_t wp[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) wp[i] = dec_pair<QBITS>(cw[j], 8 * s + i, deq[j]);
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        dec_mma(acc[j], xa[2 * b], xc[2 * b], xa[2 * b + 1], xc[2 * b + 1], wp[2 * b], wp[2 * b + 1]);
                }
            }
        }
        // every lane's reads of slot d have been used: refill it with super-stage tt + kDecD
        __syncwarp();
        issue();
    }
    // no copy may still be landing when the block exits
    for (int64_t q = waited; q < issued; ++q)
        if (!g_wait_warp(bars + 8u * (uint32_t)(q % kDecD), (uint32_t)((q / kDecD) & 1))) break;
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    if (ok) flush();
}

}  // namespace gq
