// gq_rowquant_tma.cuh -- the fused per-row kernel, pipelined through shared
// memory with bulk asynchronous copies (sm_100a).
//
// One persistent block per SM: warp 16 is the producer, warps 0..15 consume.
// The weights are cut into tiles of whole rows (one descriptor per tile) that
// fill a stage of a ring of shared-memory stages.  The producer's elected lane
// issues cp.async.bulk copies global -> shared for tile i + stages - 1 while
// the consumers work on tile i; completion is tracked by one mbarrier per
// stage ("full", transaction bytes) and stages are handed back through a
// second mbarrier ("empty", one arrival per consumer warp).  Each input byte
// is read from HBM exactly once, with up to (stages - 1) tiles in flight per SM.
//
// Consumers form teams of G warps (a power of two, per descriptor) that own a
// row: the row is read from shared memory twice (selection, then quantize),
// and every output (w_hat, int8 codes, packed int6/int8 bytes, scales) is
// written straight from registers with coalesced vector stores.
//
// Every wait is bounded (a few seconds of %globaltimer): on expiry the thread
// records GQ_STATUS_TIMEOUT in the tile's status word and leaves its loop; the
// producer first waits, again bounded, for the copies it issued.  No wait is
// expected to expire; the bound keeps a defect from hanging the GPU.
#pragma once

#include "gq_kernels.cuh"

namespace gq {

constexpr int kTmaConsumerWarps = 16;
constexpr int kTmaThreads = (kTmaConsumerWarps + 1) * 32;
constexpr int kTmaMaxStages = 4;
constexpr uint32_t kStatusTimeout = 0x4u;
constexpr unsigned long long kWaitLimitNs = 4000000000ull;   // 4 s

struct TmaParams {
    int32_t ndesc;
    int32_t nstages;
    int32_t stage_bytes;
    int32_t pad;
    int64_t start[kMaxDesc + 1];   // prefix sums of tiles
    RowDesc d[kMaxDesc];
};

// Shared memory after the stages: mbarriers, per-warp top-m lists, per-team
// radix histograms and broadcast slots.
constexpr int kTmaExtraBytes = 2 * kTmaMaxStages * 8 + kTmaConsumerWarps * kTopMax * 4 +
                               kTmaConsumerWarps * 256 * 4 + kTmaConsumerWarps * 4 * 4;

// ------------------------------------------------------------- PTX glue --

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
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
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0u && global_ns() - t0 > kWaitLimitNs) return false;
    }
}

// Bulk copy global -> this CTA's shared memory, completing `bytes` on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ float4 lds_f32x4(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(a));
    return v;
}

__device__ __forceinline__ uint2 lds_u32x2(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}

// Four consecutive elements (quad j) of a row held in shared memory.
template <int DT>
__device__ __forceinline__ void lds_quad(uint32_t row, int j, float v[4]) {
    if constexpr (DT == kF32) {
        float4 x = lds_f32x4(row + 16u * (uint32_t)j);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    } else {
        uint2 x = lds_u32x2(row + 8u * (uint32_t)j);
        v[0] = __uint_as_float(x.x << 16);
        v[1] = __uint_as_float(x.x & 0xFFFF0000u);
        v[2] = __uint_as_float(x.y << 16);
        v[3] = __uint_as_float(x.y & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

struct Team {
    int G;        // warps per team
    int team;     // team index
    int tw;       // warp index in the team
    int lane;
    int cw;       // consumer warp index
    // Named barrier ids never collide between team sizes: a warp may reach
    // the next tile (another team size) while its old teammates finish.
    //   G = 2: ids 1..8, G = 4: 9..12, G = 8: 13..14, G = 16: 15.
    __device__ __forceinline__ void sync() const {
        if (G == 1) {
            __syncwarp();
        } else {
            const int base = G == 2 ? 1 : G == 4 ? 9 : G == 8 ? 13 : 15;
            named_sync(base + team, G * 32);
        }
    }
};

// ------------------------------------------------------- row selection --

template <int DT, int M>
__device__ __forceinline__ uint2 tma_select_topm(uint32_t row, int nq, int m, const Team& T,
                                                 uint32_t* lists) {
    TopM<M> L;
    L.init();
    for (int j = T.tw * 32 + T.lane; j < nq; j += T.G * 32) {
        float v[4];
        lds_quad<DT>(row, j, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) L.insert(abs_key(v[i]));
    }
    L.warp_reduce();
    if (T.G == 1) return make_uint2(L.v[m - 1], L.v[0]);
    if (T.lane == 0) {
#pragma unroll
        for (int i = 0; i < M; ++i) lists[T.cw * kTopMax + i] = L.v[i];
    }
    T.sync();
    TopM<M> R;
    R.init();
    const int w0 = T.team * T.G;
    for (int w = 0; w < T.G; ++w) R.merge(&lists[(w0 + w) * kTopMax]);
    T.sync();
    return make_uint2(R.v[m - 1], R.v[0]);
}

// MSB-first radix select (8+8+8+7 bits) over the shared-memory row.
template <int DT>
__device__ uint32_t tma_select_radix(uint32_t row, int nq, int64_t m, const Team& T,
                                     uint32_t* hist, uint32_t* bcast, bool* nonfinite) {
    const int tt = T.tw * 32 + T.lane;
    uint32_t prefix = 0, pmask = 0;
    int64_t rem = m;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = pass == 0 ? 23 : pass == 1 ? 15 : pass == 2 ? 7 : 0;
        const uint32_t dmask = pass == 3 ? 0x7Fu : 0xFFu;
        for (int i = tt; i < 256; i += T.G * 32) hist[i] = 0u;
        T.sync();
        for (int j = tt; j < nq; j += T.G * 32) {
            float v[4];
            lds_quad<DT>(row, j, v);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t key = abs_key(v[i]);
                if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
            }
        }
        T.sync();
        if (T.tw == 0) {
            uint32_t cnt[8];
            uint32_t sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cnt[i] = hist[255 - 8 * T.lane - i];
                sum += cnt[i];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                uint32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (T.lane >= off) incl += o;
            }
            const int64_t excl = (int64_t)(incl - sum);
            if (excl < rem && rem <= excl + (int64_t)sum) {
                int64_t acc = excl;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (acc + cnt[i] >= rem) {
                        bcast[0] = (uint32_t)(255 - 8 * T.lane - i);
                        bcast[1] = (uint32_t)(rem - acc);
                        break;
                    }
                    acc += cnt[i];
                }
            }
            if (pass == 0 && T.lane == 0) bcast[2] = hist[255];
        }
        T.sync();
        const uint32_t b = bcast[0];
        rem = bcast[1];
        if (pass == 0) *nonfinite = bcast[2] != 0u;
        prefix |= b << shift;
        pmask |= dmask << shift;
        T.sync();
    }
    return prefix;
}

// ---------------------------------------------------- quantize one row --

// Quantize the four elements of a quad.  b[i] = kMagic + q[i] as a float.
// FAST: reciprocal product with the near-half guard (warp vote) instead of a
// division per element; CLIP: clip to [-c, c] first.
template <bool FAST, bool CLIP>
__device__ __forceinline__ void quantize_quad(const float v[4], const Scale& S, float b[4]) {
    float wc[4], y[4], n[4];
    bool need = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        wc[i] = CLIP ? fminf(fmaxf(v[i], -S.c), S.c) : v[i];
        y[i] = FAST ? __fmul_rn(wc[i], S.rcp) : __fdiv_rn(wc[i], S.s);
        n[i] = __fsub_rn(__fadd_rn(y[i], kMagic), kMagic);    // rint(y), exact for |y| < 2^22
        if (FAST) need |= fabsf(__fsub_rn(y[i], n[i])) > kNearHalf;
    }
    if (FAST) {
        if (__any_sync(0xFFFFFFFFu, need)) {
            if (need) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    y[i] = __fdiv_rn(wc[i], S.s);
                    n[i] = __fsub_rn(__fadd_rn(y[i], kMagic), kMagic);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float q = fminf(fmaxf(n[i], -S.qmaxf), S.qmaxf);
        b[i] = S.zero ? kMagic : __fadd_rn(q, kMagic);
    }
}

template <int DT, bool FAST, bool CLIP>
__device__ __forceinline__ void tma_quantize_row(const RowDesc& D, int64_t r, uint32_t row, int nq,
                                                 const Scale& S, const Team& T) {
    const int64_t n = D.cols;
    constexpr int esz = DT == kF32 ? 4 : 2;
    char* dqrow = D.dq ? reinterpret_cast<char*>(D.dq) + r * n * esz : nullptr;
    int8_t* crow = D.codes ? D.codes + r * n : nullptr;
    uint8_t* prow = D.packed ? D.packed + r * D.prb : nullptr;
    const bool vdq = D.flags & kVecDq;
    const bool vcodes = D.flags & kVecCodes;
    const bool vpk = D.flags & kVecPacked;
    const bool six = D.qbits == 6;
    const int lane = T.lane;

    for (int jb = T.tw * 32; jb < nq; jb += T.G * 32) {
        const int j = jb + lane;
        const bool valid = j < nq;
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        if (valid) lds_quad<DT>(row, j, v);
        float b[4];
        quantize_quad<FAST, CLIP>(v, S, b);
        const int e0 = 4 * j;
        if (valid && dqrow) {
            float d[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) d[i] = __fmul_rn(__fsub_rn(b[i], kMagic), S.s);
            if constexpr (DT == kF32) {
                float* o = reinterpret_cast<float*>(dqrow) + e0;
                if (vdq) {
                    *reinterpret_cast<float4*>(o) = make_float4(d[0], d[1], d[2], d[3]);
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) o[i] = d[i];
                }
            } else {
                uint16_t* o = reinterpret_cast<uint16_t*>(dqrow) + e0;
                uint16_t h[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) h[i] = float_to_bf16_bits(d[i]);
                if (vdq) {
                    *reinterpret_cast<uint2*>(o) = make_uint2((uint32_t)h[0] | ((uint32_t)h[1] << 16),
                                                              (uint32_t)h[2] | ((uint32_t)h[3] << 16));
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) o[i] = h[i];
                }
            }
        }
        // code bytes: the low byte of kMagic + q is q's two's-complement byte
        const uint32_t bytes4 = __byte_perm(__byte_perm(__float_as_uint(b[0]), __float_as_uint(b[1]), 0x0040),
                                            __byte_perm(__float_as_uint(b[2]), __float_as_uint(b[3]), 0x0040),
                                            0x5410);
        if (valid && crow) {
            if (vcodes) {
                *reinterpret_cast<uint32_t*>(crow + e0) = bytes4;
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) crow[e0 + i] = (int8_t)(bytes4 >> (8 * i));
            }
        }
        if (prow) {
            if (six) {
                const uint32_t v24 = (__float_as_uint(b[0]) & 63u) | ((__float_as_uint(b[1]) & 63u) << 6) |
                                     ((__float_as_uint(b[2]) & 63u) << 12) | ((__float_as_uint(b[3]) & 63u) << 18);
                const uint32_t nxt = __shfl_down_sync(0xFFFFFFFFu, v24, 1);
                const int sub = lane & 3;
                const int g0 = j - sub;
                if (valid) {
                    if (vpk && g0 + 3 < nq) {
                        if (sub < 3)
                            *reinterpret_cast<uint32_t*>(prow + 3 * g0 + 4 * sub) =
                                (v24 >> (8 * sub)) | (nxt << (24 - 8 * sub));
                    } else {
                        prow[3 * j + 0] = (uint8_t)(v24 & 0xFFu);
                        prow[3 * j + 1] = (uint8_t)((v24 >> 8) & 0xFFu);
                        prow[3 * j + 2] = (uint8_t)((v24 >> 16) & 0xFFu);
                    }
                }
            } else if (valid) {
                if (vpk) {
                    *reinterpret_cast<uint32_t*>(prow + e0) = bytes4;
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) prow[e0 + i] = (uint8_t)(bytes4 >> (8 * i));
                }
            }
        }
    }
}

template <int DT>
__device__ __forceinline__ void tma_process_row(const RowDesc& D, int64_t r, uint32_t row, const Team& T,
                                                uint32_t* lists, uint32_t* hist, uint32_t* bcast) {
    const int nq = (int)(D.cols >> 2);
    uint32_t ckey;
    bool nonfinite = false;
    if (D.clip_in) {
        ckey = *D.clip_in;
    } else {
        const int m = D.m;
        uint2 sel;
        if (m <= 1) sel = tma_select_topm<DT, 1>(row, nq, 1, T, lists);
        else if (m <= 2) sel = tma_select_topm<DT, 2>(row, nq, m, T, lists);
        else if (m <= 4) sel = tma_select_topm<DT, 4>(row, nq, m, T, lists);
        else if (m <= kTopMax) sel = tma_select_topm<DT, 8>(row, nq, m, T, lists);
        else sel = make_uint2(tma_select_radix<DT>(row, nq, m, T, hist, bcast, &nonfinite), 0u);
        ckey = sel.x;
        if (m <= kTopMax) nonfinite = sel.y >= 0x7F800000u;
    }
    uint16_t hbits;
    bool range;
    const Scale S = make_scale(ckey, D.qmax, D.export_mode != 0, &hbits, &range);
    const bool per_tensor = D.flags & kPerTensor;
    if (T.tw == 0 && T.lane == 0 && (!per_tensor || r == 0)) {
        const int64_t g = per_tensor ? 0 : r;
        if (D.clip_out) D.clip_out[g] = S.c;
        if (D.sf32) D.sf32[g] = S.s;
        if (D.sf16) D.sf16[g] = hbits;
        if (D.status) {
            const uint32_t st = (nonfinite ? kStatusNonfinite : 0u) | (range ? kStatusRange : 0u);
            if (st) atomicOr(reinterpret_cast<unsigned int*>(D.status), st);
        }
    }
    if (!(D.flags & kElemOut)) return;
    // Clipping is a no-op for the codes when the clip value itself rounds to
    // at least qmax: by monotonicity of rounded division every |w| > c then
    // also lands on +-qmax after the clamp.  Only coarse (subnormal) scales
    // need the explicit clip.
    const float cq = S.zero ? 0.f : __fsub_rn(__fadd_rn(__fdiv_rn(S.c, S.s), kMagic), kMagic);
    const bool clip = !(cq >= S.qmaxf);
    if (S.fast && !clip)
        tma_quantize_row<DT, true, false>(D, r, row, nq, S, T);
    else if (S.fast)
        tma_quantize_row<DT, true, true>(D, r, row, nq, S, T);
    else
        tma_quantize_row<DT, false, true>(D, r, row, nq, S, T);
}

// ------------------------------------------------------------- kernel --

__global__ void __launch_bounds__(kTmaThreads, 1)
rowquant_tma_kernel(const __grid_constant__ TmaParams P) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int S = P.nstages;
    const uint32_t SB = (uint32_t)P.stage_bytes;
    unsigned char* extra = smem + (size_t)S * SB;
    uint64_t* full = reinterpret_cast<uint64_t*>(extra);
    uint64_t* empty = full + kTmaMaxStages;
    uint32_t* lists = reinterpret_cast<uint32_t*>(empty + kTmaMaxStages);
    uint32_t* hist = lists + kTmaConsumerWarps * kTopMax;
    uint32_t* bcast = hist + kTmaConsumerWarps * 256;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), kTmaConsumerWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();

    const int64_t ntiles = P.start[P.ndesc];
    const uint32_t smem_base = smem_u32(smem);

    if (warp == kTmaConsumerWarps) {
        // ---------------------------------------------------- producer --
        if (lane != 0) return;
        int it = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
            const int s = it % S;
            const int k = it / S;
            const int di = find_desc(P.start, P.ndesc, t);
            const RowDesc& D = P.d[di];
            if (k > 0 && !mbar_wait(smem_u32(&empty[s]), (uint32_t)((k - 1) & 1))) {
                if (D.status) atomicOr(reinterpret_cast<unsigned int*>(D.status), kStatusTimeout);
                ok = false;
                break;
            }
            const int64_t r0 = (t - P.start[di]) * D.tile_rows;
            const int64_t nr = min((int64_t)D.tile_rows, D.rows - r0);
            const int esz = D.dtype == kF32 ? 4 : 2;
            const uint32_t row_bytes = (uint32_t)(D.cols * esz);
            const uint32_t full_bar = smem_u32(&full[s]);
            const uint32_t dst = smem_base + (uint32_t)s * SB;
            const char* src = reinterpret_cast<const char*>(D.w) + r0 * D.ld * esz;
            mbar_arrive_expect_tx(full_bar, (uint32_t)nr * row_bytes);
            if (D.ld == D.cols) {
                bulk_g2s(dst, src, (uint32_t)nr * row_bytes, full_bar);
            } else {
                for (int64_t i = 0; i < nr; ++i)
                    bulk_g2s(dst + (uint32_t)i * row_bytes, src + i * D.ld * esz, row_bytes, full_bar);
            }
        }
        if (!ok) {
            // wait (bounded) for the copies already issued before leaving
            for (int i = max(0, it - S); i < it; ++i)
                (void)mbar_wait(smem_u32(&full[i % S]), (uint32_t)((i / S) & 1));
        }
        return;
    }

    // -------------------------------------------------------- consumers --
    int it = 0;
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
        const int s = it % S;
        const int k = it / S;
        const int di = find_desc(P.start, P.ndesc, t);
        const RowDesc& D = P.d[di];
        if (!mbar_wait(smem_u32(&full[s]), (uint32_t)(k & 1))) {
            if (lane == 0 && D.status) atomicOr(reinterpret_cast<unsigned int*>(D.status), kStatusTimeout);
            break;
        }
        const int64_t r0 = (t - P.start[di]) * D.tile_rows;
        const int nr = (int)min((int64_t)D.tile_rows, D.rows - r0);
        const int esz = D.dtype == kF32 ? 4 : 2;
        const uint32_t row_bytes = (uint32_t)(D.cols * esz);
        Team T;
        T.G = D.team_warps;
        T.cw = warp;
        T.team = warp / T.G;
        T.tw = warp % T.G;
        T.lane = lane;
        const int teams = kTmaConsumerWarps / T.G;
        const uint32_t stage = smem_base + (uint32_t)s * SB;
        for (int i = T.team; i < nr; i += teams) {
            const uint32_t row = stage + (uint32_t)i * row_bytes;
            if (D.dtype == kF32)
                tma_process_row<kF32>(D, r0 + i, row, T, lists, hist + T.team * 256, bcast + T.team * 4);
            else
                tma_process_row<kBF16>(D, r0 + i, row, T, lists, hist + T.team * 256, bcast + T.team * 4);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    }
}

}  // namespace gq
