// gq_rowquant_tma.cuh -- the fused per-row kernel, pipelined through shared
// memory with bulk asynchronous copies (sm_100a).
//
// One persistent 512-thread block (16 warps) per SM and no producer warp.
// The weights are cut into tiles of whole rows (one descriptor per tile) that
// fill the stages of a ring in shared memory.  Thread 0 issues the first fill
// of every stage; after that the stage's last reader refills it:
//   - fill k of stage s completes phase k / 2 of full[2 s + k % 2] (two
//     "full" mbarriers per stage used on alternate fills, transaction bytes),
//     so a one-bit parity wait is never ambiguous for a reader that lags one
//     fill behind;
//   - done[s] counts the warps that have finished with stage s (an
//     acquire-release shared-memory atomic per warp); every fill is read by
//     one tile-team of wpt warps, so the warp whose increment makes the count
//     a multiple of wpt is the fill's last reader, and its lane 0 issues the
//     next cp.async.bulk copy into the stage.
// With three stages the 16 warps form two tile-teams of 8 that take
// alternate tiles.  Each input byte is read from HBM exactly once.
//
// A row is owned by a slot of `lpr` threads of a tile-team (lanes per row, a
// power of two from 8 to 512, chosen per descriptor):
//   lpr <= 16 : 32 / lpr rows share a warp, so every per-row step (the
//               selection butterfly, the scale, the output pointers) is one
//               warp instruction for several rows;
//   lpr >= 32 : G = lpr / 32 warps own a row; each publishes its top-m list
//               in shared memory, the row's warps meet at a named barrier and
//               every warp merges the lists.
// The row is read from shared memory twice (selection, then quantize), and
// every output (w_hat, int8 codes, packed int6 / int8 bytes, scales) is
// written from registers with coalesced vector stores.
//
// Every wait on a full barrier is bounded (4 s of %globaltimer unless the
// launch sets a shorter limit).  A warp whose wait gives up enters abort mode:
// it records GQ_STATUS_TIMEOUT in the status word of every tile it still
// touches, no longer waits, issues no refill, but still walks its
// tile-team's tiles with the same control flow, so that every named barrier
// the team meets is met by all of its warps (a warp that left would leave
// the others waiting at such a barrier forever).  Its tile-mates then give up
// at the first fill that the aborted warp would have started.  Before the
// block exits, thread 0 waits (bounded) for the last fill issued into every
// stage, so that no copy is still landing in shared memory.  No wait is
// expected to expire; the bound keeps a defect from hanging the GPU.
#pragma once

#include "gq_kernels.cuh"

namespace gq {

constexpr int kTmaConsumerWarps = 16;
constexpr int kTmaConsumers = kTmaConsumerWarps * 32;
constexpr int kTmaThreads = kTmaConsumers;   // no producer warp: consumers refill the stages
constexpr int kTmaMaxStages = 4;
constexpr uint32_t kStatusTimeout = 0x4u;
constexpr unsigned long long kWaitLimitNs = 4000000000ull;   // 4 s

// Output configurations with a branch-free inner loop (vector stores
// guaranteed by the host); anything else takes the generic loop.
constexpr int kOutDq = 1, kOutCodes = 2, kOutPacked = 4, kOutSix = 8, kOutAvg = 16;
constexpr int kOutGeneric = -1;

struct TmaParams {
    int32_t ndesc;
    int32_t nstages;
    int32_t stage_bytes;
    int32_t teams;       // tile-teams: the consumer warps split into `teams` groups
                         // that take alternate tiles (1 or 2)
    uint64_t wait_ns;    // limit of every bounded wait (kWaitLimitNs normally)
    // Test hook for the timeout path: the copy of global tile poison_tile
    // (-1: none) announces poison_bytes more bytes than it transfers, so its
    // full barrier never completes although every issued copy does.
    int64_t poison_tile;
    uint32_t poison_bytes;
    uint32_t pad_;
    int64_t start[kMaxDesc + 1];   // prefix sums of tiles
    RowDesc d[kMaxDesc];
};

// Shared memory after the stages: mbarriers and stage counters, per-warp
// selection lists, per-slot broadcast records and per-slot radix histograms.
constexpr int kBcastWords = 8;
constexpr int kTmaExtraBytes = 4 * kTmaMaxStages * 8 + 2 * kTmaConsumerWarps * kTopMax * 4 +
                               kTmaConsumerWarps * kBcastWords * 4 + kTmaConsumerWarps * 256 * 4;

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

// Shared-memory fetch-and-add with acquire-release ordering at CTA scope.
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t addr, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
    return old;
}

// Bounded wait for the completion of the phase with the given parity.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0u && global_ns() - t0 > limit_ns) return false;
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

// Four consecutive elements (quad j) of a row held in shared memory.  The
// shared-memory loads of the row kernels are plain (not volatile) asm, free
// for the compiler to schedule: every address they take derives from the
// stage address that the consumer loop launders through a volatile asm after
// the stage's barrier wait, so none can move above the wait or merge with a
// load of an earlier fill of the stage.
template <int DT>
__device__ __forceinline__ void lds_quad(uint32_t row, int j, float v[4]) {
    if constexpr (DT == kF32) {
        asm("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
                     : "r"(row + 16u * (uint32_t)j));
    } else {
        uint32_t a, b;
        asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(a), "=r"(b) : "r"(row + 8u * (uint32_t)j));
        v[0] = __uint_as_float(a << 16);
        v[1] = __uint_as_float(a & 0xFFFF0000u);
        v[2] = __uint_as_float(b << 16);
        v[3] = __uint_as_float(b & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// max that returns NaN when either input is NaN (the head of a top-m list
// carries a NaN of its row to the non-finite test).
__device__ __forceinline__ float fmax_nan(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t u) {
    return *reinterpret_cast<const __nv_bfloat162*>(&u);
}

// Two floats rounded to bf16 (nearest even), packed low / high.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Two binary32 lanes in one 64-bit register for the paired f32x2 operations.
// Each lane is a correctly rounded binary32 operation, but the code generator
// may contract a paired product with a following paired sum into one fused
// multiply-add (observed on sm_100a even with contraction disabled), so they
// serve only where a result does not depend on that (the guarded quotient).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// ------------------------------------------------------------------ slot --

// The threads that own one row.
struct Slot {
    int lpr;     // threads per row
    int slot;    // slot index among the consumers
    int tl;      // thread index within the slot
    int lane;
    int warp;    // consumer warp index
    int G;       // warps per row (lpr >= 32), else 1
    int tw;      // warp index within the slot (lpr >= 32)

    int lg;      // log2(lpr)

    __device__ __forceinline__ void init(int lanes_per_row, int w, int l) {
        lpr = lanes_per_row;
        lg = 31 - __clz(lpr);
        warp = w;
        lane = l;
        const int ct = w * 32 + l;
        slot = ct >> lg;
        tl = ct & (lpr - 1);
        G = lpr >= 32 ? lpr >> 5 : 1;
        tw = lpr >= 32 ? (w & (G - 1)) : 0;
    }
    // Named barrier ids never collide between team sizes: after a shape
    // change every consumer warp meets at barrier 0 first, and within one
    // shape each team has its own id (G = 2: 1..8, 4: 9..12, 8: 13..14, 16: 15).
    __device__ __forceinline__ void team_sync() const {
        const int base = G == 2 ? 1 : G == 4 ? 9 : G == 8 ? 13 : 15;
        named_sync(base + slot, G * 32);
    }
};

// ------------------------------------------------------- row selection --

// The M largest of a multiset of |w| (floats >= +0, compared as floats: the
// same order as their bit patterns), sorted descending (v[0] largest).
// The head v[0] is updated with a NaN-propagating max, so a NaN in the row
// ends up there; +-inf ends up there as the largest |w|.
template <int M>
struct TopMF {
    float v[M];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int i = 0; i < M; ++i) v[i] = 0.0f;
    }
    __device__ __forceinline__ void insert(float x) {
#pragma unroll
        for (int i = 0; i < M; ++i) {
            const float hi = i == 0 ? fmax_nan(v[i], x) : fmaxf(v[i], x);
            if (i + 1 < M) x = fminf(v[i], x);
            v[i] = hi;
        }
    }
    // two at a time: for M <= 2 the new top two of {v0 >= v1, a, b} are
    // max(v0, hi) and max(v1, min(v0, hi), lo) with hi / lo = max / min(a, b)
    __device__ __forceinline__ void insert2(float a, float b) {
        if constexpr (M == 1) {
            v[0] = fmax_nan(v[0], fmax_nan(a, b));
        } else if constexpr (M == 2) {
            const float hi = fmax_nan(a, b), lo = fminf(a, b);
            const float t = fminf(v[0], hi);
            v[0] = fmax_nan(v[0], hi);
            v[1] = fmaxf(v[1], fmaxf(t, lo));
        } else {
            insert(a);
            insert(b);
        }
    }
    // union with another sorted list: the (i+1)-th largest of the union is
    // max(a[i], b[i], max over j < i of min(a[j], b[i-1-j])).
    __device__ __forceinline__ void merge(const float* b) {
        float r[M];
#pragma unroll
        for (int i = 0; i < M; ++i) {
            float x = i == 0 ? fmax_nan(v[0], b[0]) : fmaxf(v[i], b[i]);
#pragma unroll
            for (int j = 0; j < i; ++j) x = fmaxf(x, fminf(v[j], b[i - 1 - j]));
            r[i] = x;
        }
#pragma unroll
        for (int i = 0; i < M; ++i) v[i] = r[i];
    }
    // merge across lanes with xor offsets from `hi` down to 1
    __device__ __forceinline__ void butterfly(int hi) {
        for (int off = hi; off >= 1; off >>= 1) {
            float o[M];
#pragma unroll
            for (int i = 0; i < M; ++i) o[i] = __shfl_xor_sync(0xFFFFFFFFu, v[i], off);
            merge(o);
        }
    }
    // the m-th largest (1 <= m <= M) without a dynamically indexed array
    __device__ __forceinline__ float get(int m) const {
        float r = v[0];
#pragma unroll
        for (int i = 1; i < M; ++i) r = (m - 1 == i) ? v[i] : r;
        return r;
    }
};

// Two interleaved top-M lists (M <= 2) of bf16 magnitudes, one per half of
// a bf16x2 register, on the packed bf16 min / max pipe (two elements per
// instruction).  bf16 values order exactly like their binary32 widening.
template <int M>
struct TopMH {
    __nv_bfloat162 v[M];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int i = 0; i < M; ++i) v[i] = as_bf162(0u);
    }
    __device__ __forceinline__ void insert2(__nv_bfloat162 a, __nv_bfloat162 b) {
        if constexpr (M == 1) {
            v[0] = __hmax2_nan(v[0], __hmax2_nan(a, b));
        } else {
            const __nv_bfloat162 hi = __hmax2_nan(a, b), lo = __hmin2(a, b);
            const __nv_bfloat162 t = __hmin2(v[0], hi);
            v[0] = __hmax2_nan(v[0], hi);
            v[1] = __hmax2(v[1], __hmax2(t, lo));
        }
    }
    // the union of both halves as one binary32 list
    __device__ __forceinline__ void to_f32(TopMF<M>& L) const {
        float lo[M], hi[M];
#pragma unroll
        for (int i = 0; i < M; ++i) {
            lo[i] = __low2float(v[i]);
            hi[i] = __high2float(v[i]);
        }
#pragma unroll
        for (int i = 0; i < M; ++i) L.v[i] = lo[i];
        L.merge(hi);
    }
};

// Per-thread top-M over the quads j = tl, tl + lpr, ... of a row.
template <int DT, int M>
__device__ __forceinline__ void topm_scan(uint32_t row, int nq, int tl, int lpr, int lg, bool rv, TopMF<M>& L) {
    constexpr uint32_t QB = DT == kF32 ? 16u : 8u;       // bytes of a quad in shared memory
    L.init();
    if (!rv) return;
    const int nfull = nq >> lg;                           // quads every thread of the slot has
    const uint32_t step = QB * (uint32_t)lpr;
    uint32_t sa = row + QB * (uint32_t)tl;
    int i = 0;
    if constexpr (DT == kBF16 && M <= 2) {
        TopMH<M> H;
        H.init();
        for (; i + 2 <= nfull; i += 2, sa += 2 * step) {
            uint32_t a0, a1, b0, b1;
            asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(a0), "=r"(a1) : "r"(sa));
            asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(b0), "=r"(b1) : "r"(sa + step));
            H.insert2(as_bf162(a0 & 0x7FFF7FFFu), as_bf162(a1 & 0x7FFF7FFFu));
            H.insert2(as_bf162(b0 & 0x7FFF7FFFu), as_bf162(b1 & 0x7FFF7FFFu));
        }
        for (int j = tl + lpr * i; j < nq; j += lpr, sa += step) {
            uint32_t a0, a1;
            asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(a0), "=r"(a1) : "r"(sa));
            H.insert2(as_bf162(a0 & 0x7FFF7FFFu), as_bf162(a1 & 0x7FFF7FFFu));
        }
        H.to_f32(L);
    } else {
        for (; i + 2 <= nfull; i += 2, sa += 2 * step) {
            float a[4], b[4];
            lds_quad<DT>(sa, 0, a);
            lds_quad<DT>(sa + step, 0, b);
#pragma unroll
            for (int k = 0; k < 4; ++k) L.insert2(fabsf(a[k]), fabsf(b[k]));
        }
        for (int j = tl + lpr * i; j < nq; j += lpr, sa += step) {
            float a[4];
            lds_quad<DT>(sa, 0, a);
#pragma unroll
            for (int k = 0; k < 4; ++k) L.insert(fabsf(a[k]));
        }
    }
}

// MSB-first radix select (8+8+8+7 bits) over the shared-memory row, for a
// team of G >= 1 whole warps (lpr >= 32).  Sets *nonfinite when a key has an
// all-ones exponent.
template <int DT>
__device__ uint32_t select_radix(uint32_t row, int nq, int64_t m, const Slot& T, uint32_t* hist,
                                 uint32_t* bc, bool* nonfinite) {
    uint32_t prefix = 0, pmask = 0;
    int64_t rem = m;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = pass == 0 ? 23 : pass == 1 ? 15 : pass == 2 ? 7 : 0;
        const uint32_t dmask = pass == 3 ? 0x7Fu : 0xFFu;
        for (int i = T.tl; i < 256; i += T.lpr) hist[i] = 0u;
        if (T.G == 1) __syncwarp(); else T.team_sync();
        for (int j = T.tl; j < nq; j += T.lpr) {
            float v[4];
            lds_quad<DT>(row, j, v);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t key = abs_key(v[i]);
                if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
            }
        }
        if (T.G == 1) __syncwarp(); else T.team_sync();
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
                const uint32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (T.lane >= off) incl += o;
            }
            const int64_t excl = (int64_t)(incl - sum);
            if (excl < rem && rem <= excl + (int64_t)sum) {
                int64_t acc = excl;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (acc + cnt[i] >= rem) {
                        bc[0] = (uint32_t)(255 - 8 * T.lane - i);
                        bc[1] = (uint32_t)(rem - acc);
                        break;
                    }
                    acc += cnt[i];
                }
            }
            if (pass == 0 && T.lane == 0) bc[2] = hist[255];
        }
        if (T.G == 1) __syncwarp(); else T.team_sync();
        const uint32_t b = bc[0];
        rem = bc[1];
        if (pass == 0) *nonfinite = bc[2] != 0u;
        prefix |= b << shift;
        pmask |= dmask << shift;
        if (T.G == 1) __syncwarp(); else T.team_sync();
    }
    return prefix;
}

// ------------------------------------------------------------ row scale --

// Everything the quantize loop needs about one row, identical in all the
// threads of its slot.
struct RowScale {
    Scale S;
    uint32_t hbits;
    bool range;
    bool nonfinite;
    bool clip;     // clip w to [-c, c] before dividing
    bool clamp;    // clamp the rounded code to [-qmax, qmax]
};

__device__ __forceinline__ void finish_scale(uint32_t ckey, bool nonfinite, const RowDesc& D, RowScale& R) {
    uint16_t h;
    R.S = make_scale(ckey, D.qmax, D.export_mode != 0, &h, &R.range);
    R.hbits = h;
    R.nonfinite = nonfinite;
    // The clip value's own code cq = rint(c / s) is exactly qmax whenever the
    // scale is a normal number: c / s32 = qmax (1 +- 2^-23), and c / h =
    // qmax (1 +- 2^-10.9) for a normal binary16 h.  Then the clip can be
    // skipped (monotone rounded division maps every |w| > c to +-qmax after
    // the clamp) and, when no |w| exceeds c (m == 1), the clamp too.
    const bool normal = D.export_mode ? ((h & 0x7C00u) != 0u && (h & 0x7C00u) != 0x7C00u)
                                      : (R.S.s >= 1.1754943508222875e-38f && R.S.s <= 3.4028234663852886e38f);
    float cq;
    if (normal) cq = R.S.qmaxf;
    else if (R.S.zero) cq = 0.0f;
    else cq = __fsub_rn(__fadd_rn(__fdiv_rn(R.S.c, R.S.s), kMagic), kMagic);
    R.clip = !(cq >= R.S.qmaxf);
    R.clamp = D.m > 1 || !(cq <= R.S.qmaxf);
}

// Per-row scalar outputs (written by thread 0 of the slot).
__device__ __forceinline__ void write_row_scalars(const RowDesc& D, int64_t r, const RowScale& R) {
    const bool per_tensor = D.flags & kPerTensor;
    if (per_tensor && r != 0) return;
    const int64_t g = per_tensor ? 0 : r;
    if (D.clip_out) D.clip_out[g] = R.S.c;
    if (D.sf32) D.sf32[g] = R.S.s;
    if (D.sf16) D.sf16[g] = (uint16_t)R.hbits;
    if (D.status) {
        const uint32_t st = (R.nonfinite ? kStatusNonfinite : 0u) | (R.range ? kStatusRange : 0u);
        if (st) atomicOr(reinterpret_cast<unsigned int*>(D.status), st);
    }
}

// ------------------------------------------------------ element kernel --

// Exact quotients for the lanes where the guard fired (rare).
__device__ __forceinline__ float4 exact_round4(float a, float b, float c, float d, float s) {
    return make_float4(__fsub_rn(__fadd_rn(__fdiv_rn(a, s), kMagic), kMagic),
                       __fsub_rn(__fadd_rn(__fdiv_rn(b, s), kMagic), kMagic),
                       __fsub_rn(__fadd_rn(__fdiv_rn(c, s), kMagic), kMagic),
                       __fsub_rn(__fadd_rn(__fdiv_rn(d, s), kMagic), kMagic));
}

__device__ __forceinline__ void exact_round8(const float* wc, float s, float* n) {
    const float4 lo = exact_round4(wc[0], wc[1], wc[2], wc[3], s);
    const float4 hi = exact_round4(wc[4], wc[5], wc[6], wc[7], s);
    n[0] = lo.x; n[1] = lo.y; n[2] = lo.z; n[3] = lo.w;
    n[4] = hi.x; n[5] = hi.y; n[6] = hi.z; n[7] = hi.w;
}

// Rounded quotients n[i] = rint(fl(wc[i] / s)) of two quads: one reciprocal
// product each, the exact division only where |y - rint(y)| > 0.5 - 2^-13
// (see kNearHalf), decided by one warp vote.
template <bool CLIP>
__device__ __forceinline__ void round8(const float x[8], const Scale& S, float n[8]) {
    float wc[8], y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        wc[i] = CLIP ? fminf(fmaxf(x[i], -S.c), S.c) : x[i];
        y[i] = __fmul_rn(wc[i], S.rcp);
        n[i] = __fsub_rn(__fadd_rn(y[i], kMagic), kMagic);
    }
    float dmax = fabsf(__fsub_rn(y[0], n[0]));
#pragma unroll
    for (int i = 1; i < 8; ++i) dmax = fmaxf(dmax, fabsf(__fsub_rn(y[i], n[i])));
    const bool need = dmax > kNearHalf;
    if (__any_sync(0xFFFFFFFFu, need)) {
        if (need) exact_round8(wc, S.s, n);
    }
}

// Rounded quotients of two quads for the branch-free loop: n[k] (integer-
// valued floats) and b[k] = kMagic + n[k] (the code bits), with one warp
// vote for both rare events: a quotient within 2^-13 of a half-integer
// (exact division for that lane) and, with CLAMP, a code beyond qmax.
// The products and sums run on element pairs (f32x2).  Whether or not the
// code generator fuses P = x * rcp into the magic sum and into the residual,
// n is rint(P) or rint(RN(P)) and e is within 2^-24 |P - n| of P - n or of
// RN(P) - n.  With Q = RN(x / s): |P - Q| < 2^-15 and |RN(P) - P| < 2^-16
// (|x / s| < 256), so |e| <= 0.5 - 2^-13 gives |Q - n| < 0.5, i.e. n = rint(Q)
// exactly, and otherwise the lane takes the exact division.
template <bool CLAMP>
__device__ __forceinline__ void round8_fast(const float x[8], float rcp, float s, float qmaxf, float n[8],
                                            float b[8]) {
    float e[8];
    const uint64_t R2 = f2_pack(rcp, rcp), M2 = f2_pack(kMagic, kMagic);
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
        const uint64_t Y = f2_mul(f2_pack(x[k], x[k + 1]), R2);
        const uint64_t B = f2_add(Y, M2);
        const uint64_t N = f2_sub(B, M2);
        f2_unpack(f2_sub(Y, N), e[k], e[k + 1]);
        f2_unpack(B, b[k], b[k + 1]);
        f2_unpack(N, n[k], n[k + 1]);
    }
    float dmax = fabsf(e[0]);
#pragma unroll
    for (int k = 1; k < 8; ++k) dmax = fmaxf(dmax, fabsf(e[k]));
    const bool near = dmax > kNearHalf;
    bool rare = near;
    if (CLAMP) {
        float nmax = fabsf(n[0]);
#pragma unroll
        for (int k = 1; k < 8; ++k) nmax = fmaxf(nmax, fabsf(n[k]));
        rare |= nmax > qmaxf;
    }
    if (__any_sync(0xFFFFFFFFu, rare)) {
        if (near) exact_round8(x, s, n);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (CLAMP) n[k] = fminf(fmaxf(n[k], -qmaxf), qmaxf);
            b[k] = __fadd_rn(n[k], kMagic);
        }
    }
}

// (0x4B400000 - 32) * (1 + 64 + 4096 + 262144) mod 2^32: the offset that
// turns the sum of four code words b into the biased 24-bit group.
constexpr uint32_t kSixBias = 0x1ABDF7E0u;

// New averages of a quad.  Scalar explicit-rounding operations: every step
// must round on its own here (the paired f32x2 forms may be contracted into
// fused multiply-adds by the code generator).
__device__ __forceinline__ float4 avg_quad(const float4 a, const float x[4], const AvgOp& A) {
    return make_float4(avg_update(a.x, x[0], A), avg_update(a.y, x[1], A), avg_update(a.z, x[2], A),
                       avg_update(a.w, x[3], A));
}

// Stores of one quad for a compile-time output configuration, at running
// pointers: pd (w_hat quad), pc (4 code bytes), pp (int8: 4 bytes; int6: this
// lane's 32-bit word of its 4-lane group, unused by the group's 4th lane), pa
// (the quad's averages, whose old values a4 the caller loaded early).
// b[i] = kMagic + q[i]: its low byte is q's two's-complement byte and its low
// six bits the int6 field.
template <int DT, int OUT>
__device__ __forceinline__ void put_quad(char* pd, int8_t* pc, uint8_t* pp, float* pa, float4 a4,
                                         const AvgOp& A, bool valid, int sub, const float q[4],
                                         const float b[4], float s) {
    const uint32_t b0 = __float_as_uint(b[0]), b1 = __float_as_uint(b[1]);
    const uint32_t b2 = __float_as_uint(b[2]), b3 = __float_as_uint(b[3]);
    if constexpr ((OUT & (kOutDq | kOutAvg)) != 0) {
        float w[4];
        const uint64_t S2 = f2_pack(s, s);
        f2_unpack(f2_mul(f2_pack(q[0], q[1]), S2), w[0], w[1]);
        f2_unpack(f2_mul(f2_pack(q[2], q[3]), S2), w[2], w[3]);
        uint2 d;
        if constexpr (DT == kBF16) d = make_uint2(pack_bf16x2(w[0], w[1]), pack_bf16x2(w[2], w[3]));
        if constexpr ((OUT & kOutDq) != 0) {
            if constexpr (DT == kF32) {
                if (valid) *reinterpret_cast<float4*>(pd) = make_float4(w[0], w[1], w[2], w[3]);
            } else {
                if (valid) *reinterpret_cast<uint2*>(pd) = d;
            }
        }
        if constexpr ((OUT & kOutAvg) != 0) {
            // the snapshot as the model holds it: RN(q * s), bf16 w_hat widened
            float x[4] = {__fmul_rn(q[0], s), __fmul_rn(q[1], s), __fmul_rn(q[2], s), __fmul_rn(q[3], s)};
            if constexpr (DT == kBF16) {
                x[0] = __uint_as_float(d.x << 16);
                x[1] = __uint_as_float(d.x & 0xFFFF0000u);
                x[2] = __uint_as_float(d.y << 16);
                x[3] = __uint_as_float(d.y & 0xFFFF0000u);
            }
            const float4 r = avg_quad(a4, x, A);
            if (valid) *reinterpret_cast<float4*>(pa) = r;
        }
    }
    if constexpr ((OUT & kOutCodes) != 0 || ((OUT & kOutPacked) != 0 && (OUT & kOutSix) == 0)) {
        const uint32_t bytes4 = __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
        if constexpr ((OUT & kOutCodes) != 0) {
            if (valid) *reinterpret_cast<uint32_t*>(pc) = bytes4;
        }
        if constexpr ((OUT & kOutPacked) != 0 && (OUT & kOutSix) == 0) {
            if (valid) *reinterpret_cast<uint32_t*>(pp) = bytes4;
        }
    }
    if constexpr ((OUT & kOutPacked) != 0 && (OUT & kOutSix) != 0) {
        // The 24-bit group of the quad without per-field masks: u = q + 32 is
        // in [1, 63], so U = u0 + 64 u1 + 4096 u2 + 262144 u3 has no carries
        // between fields, and a code's two's-complement field is u ^ 32.  As
        // integers b = 0x4B400000 + q, so U = b0 + 64 b1 + 4096 b2 + 262144 b3
        // - kSixBias (mod 2^32).
        const uint32_t v24 = ((b0 + 64u * b1 + 4096u * b2 + 262144u * b3) - kSixBias) ^ 0x820820u;
        // four lanes pack 16 codes into three aligned 32-bit words: word sub
        // is bytes 3 sub .. 3 sub + 3 of the group pair (this lane, next lane)
        const uint32_t nxt = __shfl_down_sync(0xFFFFFFFFu, v24, 1);
        const uint32_t word = __byte_perm(v24, nxt, (uint32_t)(0x654254214210ull >> (16 * sub)) & 0xFFFFu);
        if (valid && sub < 3) *reinterpret_cast<uint32_t*>(pp) = word;
    }
}

// Branch-free loop for a common output configuration: reciprocal path, no
// clip (normal scale), CLAMP when some |w| may exceed c.  All stores are
// vectorised (the host checked the alignment), all int6 groups are full.
// Full trips (two quads every thread of the slot has) run without any
// per-lane test; stores are predicated on rv (an idle sub-warp slot reads a
// valid row and writes nothing).
template <int DT, int OUT, bool CLAMP>
__device__ __forceinline__ void quantize_row_fast(uint32_t row, int nq, int tl, int lpr, int lg, bool rv,
                                                  float s, float rcp, float qmaxf, char* dq, int8_t* codes,
                                                  uint8_t* packed, const AvgOp& A) {
    constexpr uint32_t QB = DT == kF32 ? 16u : 8u;
    constexpr int DQB = DT == kF32 ? 16 : 8;
    constexpr bool SIX = (OUT & kOutSix) != 0;
    constexpr bool AVG = (OUT & kOutAvg) != 0;
    const int sub = tl & 3;
    float* pa = AVG ? A.a + 4 * tl : nullptr;          // averages: 16 bytes per quad
    const int sa4 = 4 * lpr;
    const uint32_t step = QB * (uint32_t)lpr;
    uint32_t sa = row + QB * (uint32_t)tl;
    char* pd = dq + DQB * tl;
    int8_t* pc = codes + 4 * tl;
    uint8_t* pp = packed + (SIX ? 3 * (tl - sub) + 4 * sub : 4 * tl);
    const int sd = DQB * lpr, sc = 4 * lpr, sp = SIX ? 3 * lpr : 4 * lpr;
    const int nfull = nq >> lg;
    int i = 0;
    for (; i + 2 <= nfull; i += 2) {
        float x[8];
        lds_quad<DT>(sa, 0, x);
        lds_quad<DT>(sa + step, 0, x + 4);
        float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
        if (AVG && rv) {                               // issued before the arithmetic
            a0 = *reinterpret_cast<const float4*>(pa);
            a1 = *reinterpret_cast<const float4*>(pa + sa4);
        }
        // only codes of |w| > c can exceed qmax, so the clamp is a rare path
        float q[8], b[8];
        round8_fast<CLAMP>(x, rcp, s, qmaxf, q, b);
        put_quad<DT, OUT>(pd, pc, pp, pa, a0, A, rv, sub, q, b, s);
        put_quad<DT, OUT>(pd + sd, pc + sc, pp + sp, AVG ? pa + sa4 : nullptr, a1, A, rv, sub, q + 4, b + 4, s);
        sa += 2 * step;
        pd += 2 * sd;
        pc += 2 * sc;
        pp += 2 * sp;
        if (AVG) pa += 2 * sa4;
    }
    const int niter = (nq + lpr - 1) >> lg;
    for (; i < niter; ++i) {
        const bool valid = rv && (tl + lpr * i < nq);
        float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (valid) lds_quad<DT>(sa, 0, x);
        float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (AVG && valid) a0 = *reinterpret_cast<const float4*>(pa);
        float q[8], b[8];
        round8_fast<CLAMP>(x, rcp, s, qmaxf, q, b);
        put_quad<DT, OUT>(pd, pc, pp, pa, a0, A, valid, sub, q, b, s);
        sa += step;
        pd += sd;
        pc += sc;
        pp += sp;
        if (AVG) pa += sa4;
    }
}

// Generic loop: any output configuration and alignment, coarse scales (clip),
// scales outside the reciprocal range (division per element), s == 0.
template <int DT>
__device__ __forceinline__ void quantize_row_generic(uint32_t row, int nq, int tl, int lpr, bool rv, float c,
                                                  float s, float rcp, float qmaxf, bool fast, bool zero,
                                                  bool clip, bool clamp, char* dq, int8_t* codes,
                                                  uint8_t* packed, bool vdq, bool vcodes, bool vpk, bool six,
                                                  const AvgOp& A) {
    Scale S;
    S.c = c;
    S.s = s;
    S.rcp = rcp;
    S.qmaxf = qmaxf;
    S.fast = fast;
    S.zero = zero;
    struct {
        bool clip, clamp;
    } R = {clip, clamp};
    struct {
        int tl, lpr;
    } T = {tl, lpr};
    const int niter = (nq + T.lpr - 1) >> (31 - __clz(T.lpr));
    for (int i = 0; i < niter; ++i) {
        const int j = T.tl + T.lpr * i;
        const bool valid = rv && j < nq;
        float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (valid) lds_quad<DT>(row, j, x);
        // Rows of one warp may differ in mode (zero scale, reciprocal path,
        // exact division): every lane computes with per-lane selects so the
        // warp vote below is reached by all 32 lanes.
        float wc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float nn[8];
        float dmax = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            wc[k] = R.clip ? fminf(fmaxf(x[k], -S.c), S.c) : x[k];
            const float y = S.fast ? __fmul_rn(wc[k], S.rcp) : 0.0f;
            nn[k] = __fsub_rn(__fadd_rn(y, kMagic), kMagic);
            dmax = fmaxf(dmax, fabsf(__fsub_rn(y, nn[k])));
        }
        const bool need = !S.zero && (!S.fast || dmax > kNearHalf);
        if (__any_sync(0xFFFFFFFFu, need)) {
            if (need) exact_round8(wc, S.s, nn);
        }
        float q[4], b[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            q[k] = R.clamp ? fminf(fmaxf(nn[k], -S.qmaxf), S.qmaxf) : nn[k];
            if (S.zero) q[k] = 0.0f;
            b[k] = __fadd_rn(q[k], kMagic);
        }
        const int e0 = 4 * j;
        if (valid && A.a) {
            // the snapshot as the model holds it (bf16 w_hat widened)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float x = __fmul_rn(q[k], S.s);
                if (DT == kBF16) x = bf16_bits_to_float(float_to_bf16_bits(x));
                A.a[e0 + k] = avg_update(A.a[e0 + k], x, A);
            }
        }
        if (valid && dq) {
            float d[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) d[k] = __fmul_rn(q[k], S.s);
            if (DT == kF32) {
                float* o = reinterpret_cast<float*>(dq) + e0;
                if (vdq) {
                    *reinterpret_cast<float4*>(o) = make_float4(d[0], d[1], d[2], d[3]);
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) o[k] = d[k];
                }
            } else {
                uint16_t* o = reinterpret_cast<uint16_t*>(dq) + e0;
                uint16_t h[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) h[k] = float_to_bf16_bits(d[k]);
                if (vdq) {
                    *reinterpret_cast<uint2*>(o) = make_uint2((uint32_t)h[0] | ((uint32_t)h[1] << 16),
                                                              (uint32_t)h[2] | ((uint32_t)h[3] << 16));
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) o[k] = h[k];
                }
            }
        }
        const uint32_t b0 = __float_as_uint(b[0]), b1 = __float_as_uint(b[1]);
        const uint32_t b2 = __float_as_uint(b[2]), b3 = __float_as_uint(b[3]);
        const uint32_t bytes4 = __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
        if (valid && codes) {
            if (vcodes) {
                *reinterpret_cast<uint32_t*>(codes + e0) = bytes4;
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k) codes[e0 + k] = (int8_t)(bytes4 >> (8 * k));
            }
        }
        if (packed && six) {
            const uint32_t v24 = (b0 & 0x3Fu) | ((b1 << 6) & 0xFC0u) | ((b2 << 12) & 0x3F000u) | ((b3 << 18) & 0xFC0000u);
            const uint32_t nxt = __shfl_down_sync(0xFFFFFFFFu, v24, 1);
            const int sub = T.tl & 3;
            const int g0 = j - sub;
            // the group is stored as words only when its four quads exist
            const bool gfull = g0 + 3 < nq;
            if (valid) {
                if (vpk && gfull) {
                    if (sub < 3)
                        *reinterpret_cast<uint32_t*>(packed + 3 * g0 + 4 * sub) = (v24 >> (8 * sub)) | (nxt << (24 - 8 * sub));
                } else {
                    packed[3 * j + 0] = (uint8_t)(v24 & 0xFFu);
                    packed[3 * j + 1] = (uint8_t)((v24 >> 8) & 0xFFu);
                    packed[3 * j + 2] = (uint8_t)((v24 >> 16) & 0xFFu);
                }
            }
        } else if (packed && valid) {
            if (vpk) {
                *reinterpret_cast<uint32_t*>(packed + e0) = bytes4;
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k) packed[e0 + k] = (uint8_t)(bytes4 >> (8 * k));
            }
        }
    }
}

template <int DT, int OUT>
__device__ __forceinline__ void dispatch_fast(bool clamp, uint32_t row, int nq, int tl, int lpr, bool rv,
                                              const Scale& S, char* dq, int8_t* codes, uint8_t* packed,
                                              const AvgOp& A) {
    const int lg = 31 - __clz(lpr);
    if (clamp) quantize_row_fast<DT, OUT, true>(row, nq, tl, lpr, lg, rv, S.s, S.rcp, S.qmaxf, dq, codes, packed, A);
    else quantize_row_fast<DT, OUT, false>(row, nq, tl, lpr, lg, rv, S.s, S.rcp, S.qmaxf, dq, codes, packed, A);
}

// Quantize + outputs of one row; `rv` false for an idle sub-warp slot (it
// still takes part in the warp's shuffles and votes).
template <int DT>
__device__ __forceinline__ void quantize_row(const RowDesc& D, int64_t r, uint32_t row, int nq, const Slot& T,
                                             bool rv, const RowScale& R) {
    const int out = D.out_mode;
    constexpr int esz = DT == kF32 ? 4 : 2;
    char* dq = D.dq ? reinterpret_cast<char*>(D.dq) + r * D.cols * esz : nullptr;
    int8_t* codes = D.codes ? D.codes + r * D.cols : nullptr;
    uint8_t* packed = D.packed ? D.packed + r * D.prb : nullptr;
    const AvgOp A{D.avg ? D.avg + r * D.cols : nullptr, D.avg_t, D.avg_c, D.avg_kind};
    // a warp takes the branch-free loop only if every row it holds can; the
    // clamp decision must agree too (it is a template parameter there)
    const bool fast_row = out != kOutGeneric && R.S.fast && !R.S.zero && !R.clip;
    const bool all_fast = __all_sync(0xFFFFFFFFu, fast_row || !rv);
    const bool any_clamp = __any_sync(0xFFFFFFFFu, rv && R.clamp);
    if (!all_fast) {
        quantize_row_generic<DT>(row, nq, T.tl, T.lpr, rv, R.S.c, R.S.s, R.S.rcp, R.S.qmaxf, R.S.fast, R.S.zero,
                                 R.clip, R.clamp, dq, codes, packed, (D.flags & kVecDq) != 0,
                                 (D.flags & kVecCodes) != 0, (D.flags & kVecPacked) != 0, D.qbits == 6, A);
        return;
    }
    switch (out) {
        case kOutDq | kOutPacked | kOutSix:
            dispatch_fast<DT, kOutDq | kOutPacked | kOutSix>(any_clamp, row, nq, T.tl, T.lpr, rv, R.S, dq, codes, packed, A); break;
        case kOutDq | kOutPacked:
            dispatch_fast<DT, kOutDq | kOutPacked>(any_clamp, row, nq, T.tl, T.lpr, rv, R.S, dq, codes, packed, A); break;
        case kOutDq:
            dispatch_fast<DT, kOutDq>(any_clamp, row, nq, T.tl, T.lpr, rv, R.S, dq, codes, packed, A); break;
        case kOutPacked | kOutSix:
            dispatch_fast<DT, kOutPacked | kOutSix>(any_clamp, row, nq, T.tl, T.lpr, rv, R.S, dq, codes, packed, A); break;
        case kOutPacked:
            dispatch_fast<DT, kOutPacked>(any_clamp, row, nq, T.tl, T.lpr, rv, R.S, dq, codes, packed, A); break;
        case kOutDq | kOutCodes | kOutPacked | kOutSix:
            dispatch_fast<DT, kOutDq | kOutCodes | kOutPacked | kOutSix>(any_clamp, row, nq, T.tl, T.lpr, rv, R.S, dq, codes, packed, A); break;
        case kOutAvg:
            dispatch_fast<DT, kOutAvg>(any_clamp, row, nq, T.tl, T.lpr, rv, R.S, dq, codes, packed, A); break;
        case kOutDq | kOutAvg:
            dispatch_fast<DT, kOutDq | kOutAvg>(any_clamp, row, nq, T.tl, T.lpr, rv, R.S, dq, codes, packed, A); break;
        default:
            dispatch_fast<DT, kOutDq | kOutCodes>(any_clamp, row, nq, T.tl, T.lpr, rv, R.S, dq, codes, packed, A); break;
    }
}

// ---------------------------------------------------------------- rows --

// A row owned by lpr <= 32 threads of one warp (32 / lpr rows per warp).
// The host routes rows that need the radix select (m > kTopMax) to whole
// warps, so here m <= kTopMax.
template <int DT>
__device__ __forceinline__ void process_row_sub(const RowDesc& D, int64_t r, uint32_t row, const Slot& T, bool rv) {
    const int nq = (int)(D.cols >> 2);
    uint32_t ckey;
    bool nonfinite = false;
    if (D.clip_in) {
        ckey = *D.clip_in;
    } else {
        const int m = D.m;
        float sel, top;
        if (m <= 1) {
            TopMF<1> L; topm_scan<DT, 1>(row, nq, T.tl, T.lpr, T.lg, rv, L); L.butterfly(T.lpr >> 1);
            sel = L.v[0]; top = L.v[0];
        } else if (m <= 2) {
            TopMF<2> L; topm_scan<DT, 2>(row, nq, T.tl, T.lpr, T.lg, rv, L); L.butterfly(T.lpr >> 1);
            sel = L.get(m); top = L.v[0];
        } else if (m <= 4) {
            TopMF<4> L; topm_scan<DT, 4>(row, nq, T.tl, T.lpr, T.lg, rv, L); L.butterfly(T.lpr >> 1);
            sel = L.get(m); top = L.v[0];
        } else {
            TopMF<8> L; topm_scan<DT, 8>(row, nq, T.tl, T.lpr, T.lg, rv, L); L.butterfly(T.lpr >> 1);
            sel = L.get(m); top = L.v[0];
        }
        ckey = __float_as_uint(sel);
        nonfinite = !(top <= 3.4028234663852886e38f);
    }
    RowScale R;
    finish_scale(ckey, nonfinite, D, R);
    if (rv && T.tl == 0) write_row_scalars(D, r, R);
    if (D.flags & kElemOut) quantize_row<DT>(D, r, row, nq, T, rv, R);
}

// Per-warp top-M of a team row, merged by every warp of the team; returns
// the m-th largest and whether the row holds a non-finite value.  The lists
// are double-buffered on the parity of the team's row sequence number, so
// one team barrier per row suffices: a list slot is rewritten two rows
// later, after a barrier every reader has passed.
template <int DT, int M>
__device__ __forceinline__ void team_topm(uint32_t row, int nq, int m, const Slot& T, float* lists, int seq,
                                          uint32_t* ckey, bool* nonfinite) {
    TopMF<M> L;
    topm_scan<DT, M>(row, nq, T.tl, T.lpr, T.lg, true, L);
    L.butterfly(16);
    if (T.G > 1) {
        float* buf = lists + (seq & 1) * (kTmaConsumerWarps * kTopMax);
        if (T.lane == 0) {
#pragma unroll
            for (int i = 0; i < M; ++i) buf[T.warp * kTopMax + i] = L.v[i];
        }
        T.team_sync();
        L.init();
        if (T.lane < T.G) {
            const float* src = buf + (T.slot * T.G + T.lane) * kTopMax;
#pragma unroll
            for (int i = 0; i < M; ++i) L.v[i] = src[i];
        }
        L.butterfly(T.G >> 1);
#pragma unroll
        for (int i = 0; i < M; ++i) L.v[i] = __shfl_sync(0xFFFFFFFFu, L.v[i], 0);
    }
    *ckey = __float_as_uint(L.get(m));
    *nonfinite = !(L.v[0] <= 3.4028234663852886e38f);
}

// A row owned by G >= 1 whole warps.
template <int DT>
__device__ __forceinline__ void process_row_team(const RowDesc& D, int64_t r, uint32_t row, const Slot& T,
                                                 float* lists, uint32_t* bc, uint32_t* hist, int seq) {
    const int nq = (int)(D.cols >> 2);
    const int m = D.m;
    uint32_t ckey;
    bool nonfinite = false;
    if (D.clip_in) ckey = *D.clip_in;
    else if (m > kTopMax) ckey = select_radix<DT>(row, nq, m, T, hist, bc, &nonfinite);
    else if (m <= 1) team_topm<DT, 1>(row, nq, 1, T, lists, seq, &ckey, &nonfinite);
    else if (m <= 2) team_topm<DT, 2>(row, nq, m, T, lists, seq, &ckey, &nonfinite);
    else if (m <= 4) team_topm<DT, 4>(row, nq, m, T, lists, seq, &ckey, &nonfinite);
    else team_topm<DT, 8>(row, nq, m, T, lists, seq, &ckey, &nonfinite);
    RowScale R;
    finish_scale(ckey, nonfinite, D, R);
    if (T.tl == 0) write_row_scalars(D, r, R);
    if (D.flags & kElemOut) quantize_row<DT>(D, r, row, nq, T, true, R);
}

// ------------------------------------------------------------- kernel --

// Start the bulk copy of this CTA's tile number `it` (global tile
// blockIdx.x + it * gridDim.x) into stage it % S as fill it / S of that
// stage.  `di` is the caller's descriptor cursor: tiles it issues only grow.
__device__ __forceinline__ void issue_tile(const TmaParams& P, int it, int& di, uint32_t smem_base, uint32_t SB,
                                           int S, uint32_t bar) {
    const int64_t t = blockIdx.x + (int64_t)it * gridDim.x;
    while (t >= P.start[di + 1]) ++di;
    const RowDesc& D = P.d[di];
    const int64_t r0 = (t - P.start[di]) * D.tile_rows;
    const int64_t nr = min((int64_t)D.tile_rows, D.rows - r0);
    const int esz = D.dtype == kF32 ? 4 : 2;
    const uint32_t row_bytes = (uint32_t)(D.cols * esz);
    const uint32_t dst = smem_base + (uint32_t)(it % S) * SB;
    const char* src = reinterpret_cast<const char*>(D.w) + r0 * D.ld * esz;
    mbar_arrive_expect_tx(bar, (uint32_t)nr * row_bytes + (t == P.poison_tile ? P.poison_bytes : 0u));
    if (D.ld == D.cols) {
        bulk_g2s(dst, src, (uint32_t)nr * row_bytes, bar);
    } else {
        for (int64_t i = 0; i < nr; ++i) bulk_g2s(dst + (uint32_t)i * row_bytes, src + i * D.ld * esz, row_bytes, bar);
    }
}

// AWQ column scaling of one staged row, in place: element c becomes
// RN_dtype(w * t[c]) -- one binary32 multiply, rounded to nearest even bf16
// for a bf16 weight.  Thread `tl` of the row's `lpr` threads takes quads
// tl, tl + lpr, ... (cols a multiple of 4), kScaleBatch at a time: the
// batch's scale loads and shared-memory loads are all issued before its
// first store, so their latencies overlap instead of adding up quad by quad.
// The shared-memory accesses are volatile (kept in program order, loads of a
// batch before its stores) but carry no memory clobber, so the scale loads
// are free to move ahead of them.  Each thread touches only its own quads.
// The caller syncs the row's threads before they read the row, after the
// proxy fence here that orders these generic stores before the next bulk
// copy into the stage.
constexpr int kScaleBatch = 8;

__device__ __forceinline__ void scale_quad_f32(uint32_t a, float4 c) {
    float v0, v1, v2, v3;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v0), "=f"(v1), "=f"(v2), "=f"(v3) : "r"(a));
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(__fmul_rn(v0, c.x)),
                 "f"(__fmul_rn(v1, c.y)), "f"(__fmul_rn(v2, c.z)), "f"(__fmul_rn(v3, c.w)));
}

__device__ __forceinline__ uint32_t scale_pair_bf16(uint32_t x, float c0, float c1) {
    const __nv_bfloat162 r = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(x << 16), c0),
                                                   __fmul_rn(__uint_as_float(x & 0xFFFF0000u), c1));
    return *reinterpret_cast<const uint32_t*>(&r);
}

__device__ __forceinline__ void scale_row(uint32_t row, int cols, int dtype, const float* t, int tl, int lpr) {
    const int qpr = cols >> 2;
    const float4* t4 = reinterpret_cast<const float4*>(t);
    int j = tl;
    if (dtype == kF32) {
        for (; j + (kScaleBatch - 1) * lpr < qpr; j += kScaleBatch * lpr) {
            float4 c[kScaleBatch];
            float v[kScaleBatch][4];
#pragma unroll
            for (int b = 0; b < kScaleBatch; ++b) c[b] = __ldg(t4 + j + b * lpr);
#pragma unroll
            for (int b = 0; b < kScaleBatch; ++b)
                asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                             : "=f"(v[b][0]), "=f"(v[b][1]), "=f"(v[b][2]), "=f"(v[b][3])
                             : "r"(row + 16u * (uint32_t)(j + b * lpr)));
#pragma unroll
            for (int b = 0; b < kScaleBatch; ++b)
                asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(row + 16u * (uint32_t)(j + b * lpr)),
                             "f"(__fmul_rn(v[b][0], c[b].x)), "f"(__fmul_rn(v[b][1], c[b].y)),
                             "f"(__fmul_rn(v[b][2], c[b].z)), "f"(__fmul_rn(v[b][3], c[b].w)));
        }
        for (; j < qpr; j += lpr) scale_quad_f32(row + 16u * (uint32_t)j, __ldg(t4 + j));
    } else {
        for (; j + (kScaleBatch - 1) * lpr < qpr; j += kScaleBatch * lpr) {
            float4 c[kScaleBatch];
            uint32_t x[kScaleBatch], y[kScaleBatch];
#pragma unroll
            for (int b = 0; b < kScaleBatch; ++b) c[b] = __ldg(t4 + j + b * lpr);
#pragma unroll
            for (int b = 0; b < kScaleBatch; ++b)
                asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                             : "=r"(x[b]), "=r"(y[b]) : "r"(row + 8u * (uint32_t)(j + b * lpr)));
#pragma unroll
            for (int b = 0; b < kScaleBatch; ++b)
                asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(row + 8u * (uint32_t)(j + b * lpr)),
                             "r"(scale_pair_bf16(x[b], c[b].x, c[b].y)), "r"(scale_pair_bf16(y[b], c[b].z, c[b].w)));
        }
        for (; j < qpr; j += lpr) {
            const float4 c = __ldg(t4 + j);
            const uint32_t a = row + 8u * (uint32_t)j;
            uint32_t x, y;
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(x), "=r"(y) : "r"(a));
            asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(scale_pair_bf16(x, c.x, c.y)),
                         "r"(scale_pair_bf16(y, c.z, c.w)));
        }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// The row's address after its in-place rescale and the sync that follows:
// passed through a volatile asm placed after the sync, so that no read of the
// rescaled row (plain asm loads, free to move) can be scheduled above it.
__device__ __forceinline__ uint32_t launder_row(uint32_t row) {
    uint32_t r;
    asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(row) : "memory");
    return r;
}

// kColScale: the launch's descriptors all carry AWQ column scales (a
// separate instantiation keeps the plain kernel's code untouched).
template <bool kColScale>
__global__ void __launch_bounds__(kTmaThreads, 1)
rowquant_tma_kernel(const __grid_constant__ TmaParams P) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int S = P.nstages;
    const uint32_t SB = (uint32_t)P.stage_bytes;
    unsigned char* extra = smem + (size_t)S * SB;
    // Two "full" barriers per stage, used on alternate fills: fill k of stage
    // s completes phase k / 2 of full[2 s + k % 2].  A tile-team lags at most
    // one fill of a stage behind (the other team's tile), and a one-bit
    // parity wait stays unambiguous only while the waiter is less than two
    // phases of its barrier behind, which alternation guarantees.
    uint64_t* full = reinterpret_cast<uint64_t*>(extra);
    // done[s]: warps that have finished with stage s, over all its fills.
    // Every fill is read by one tile-team of wpt warps, so the warp whose
    // increment makes the count a multiple of wpt is the last reader of the
    // fill and starts the next one.
    uint32_t* done = reinterpret_cast<uint32_t*>(full + 2 * kTmaMaxStages);
    // last_fill[s]: the latest fill issued into stage s (-1: none), and the
    // count of warps that have left the tile loop, for the drain before exit
    int32_t* last_fill = reinterpret_cast<int32_t*>(done + kTmaMaxStages);
    uint32_t* exited = reinterpret_cast<uint32_t*>(last_fill + kTmaMaxStages);
    auto full_bar = [&](int stage, int fill) { return smem_u32(&full[2 * stage + (fill & 1)]); };
    auto full_parity = [](int fill) { return (uint32_t)((fill >> 1) & 1); };
    float* lists = reinterpret_cast<float*>(full + 4 * kTmaMaxStages);                     // [2][warp][kTopMax]
    uint32_t* bcast = reinterpret_cast<uint32_t*>(lists + 2 * kTmaConsumerWarps * kTopMax);  // [slot][8]
    uint32_t* hist = bcast + kTmaConsumerWarps * kBcastWords;                          // [slot][256]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t ntiles = P.start[P.ndesc];
    const uint32_t smem_base = smem_u32(smem);
    int di_issue = 0;     // descriptor cursor of the tiles this thread issues
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[2 * s]), 1);
            mbar_init(smem_u32(&full[2 * s + 1]), 1);
            done[s] = 0u;
            last_fill[s] = blockIdx.x + (int64_t)s * gridDim.x < ntiles ? 0 : -1;
        }
        *exited = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        // first fill of every stage
        for (int it = 0; it < S && blockIdx.x + (int64_t)it * gridDim.x < ntiles; ++it)
            issue_tile(P, it, di_issue, smem_base, SB, S, full_bar(it, 0));
    }
    __syncthreads();

    // Tile-team `team` takes the tiles it == team (mod teams); its slots are
    // numbered globally (slot = thread / lpr), so the shared records of
    // different tile-teams never overlap.
    const int teams = P.teams;
    const int wpt = kTmaConsumerWarps / teams;       // warps per tile-team
    const int team = warp / wpt;
    const int team_threads = wpt * 32;
    int it = 0;
    int di = 0;           // tiles come in increasing order: their descriptors too
    int prev_lpr = 0;
    int seq = 0;          // rows this warp's slot has processed since the last shape change
    bool aborted = false; // a wait of this warp gave up (warp-uniform)
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
        if (it % teams != team) continue;
        const int s = it % S;
        const int k = it / S;
        while (t >= P.start[di + 1]) ++di;
        const RowDesc& D = P.d[di];
        const int lpr = D.lanes_per_row;
        if (lpr != prev_lpr) {
            // the slot shape changes: no warp of this tile-team may still use
            // the old slots' shared records (all its warps take this branch on
            // the same tile); team 0 meets at barrier 0, team 1 at barrier 15
            // (free: a 16-warp row needs a single tile-team)
            if (prev_lpr != 0) named_sync(team == 0 ? 0 : 15, team_threads);
            prev_lpr = lpr;
            seq = 0;
        }
        if (!aborted) aborted = !__all_sync(0xFFFFFFFFu, mbar_wait(full_bar(s, k), full_parity(k), P.wait_ns));
        // abort mode: the tile is walked with the team (its barriers are met)
        // but its stage may hold anything; its outputs are marked unspecified
        if (aborted && lane == 0 && D.status) atomicOr(reinterpret_cast<unsigned int*>(D.status), kStatusTimeout);
        const int64_t r0 = (t - P.start[di]) * D.tile_rows;
        const int nr = (int)min((int64_t)D.tile_rows, D.rows - r0);
        const uint32_t row_bytes = (uint32_t)(D.cols * (D.dtype == kF32 ? 4 : 2));
        uint32_t stage;   // opaque to the compiler, ordered after the wait (see lds_quad)
        asm volatile("mov.b32 %0, %1;" : "=r"(stage) : "r"(smem_base + (uint32_t)s * SB) : "memory");
        Slot T;
        T.init(lpr, warp, lane);
        const int slots = team_threads >> T.lg;          // slots of this tile-team
        const int lslot = T.slot - team * slots;         // slot index within it
        if (lpr < 32) {
            const int rounds = (nr + slots - 1) / slots;
            for (int rd = 0; rd < rounds; ++rd) {
                const int i = rd * slots + lslot;
                const bool rv = i < nr;
                const uint32_t row = stage + (uint32_t)(rv ? i : 0) * row_bytes;
                uint32_t srow = row;
                if constexpr (kColScale) {
                    // AWQ: the row becomes RN_dtype(w * t[c]) in place before its
                    // threads read it (the slots of a warp run in lockstep)
                    if (rv) scale_row(row, (int)D.cols, D.dtype, D.colscale, T.tl, lpr);
                    __syncwarp();
                    srow = launder_row(row);
                }
                if (D.dtype == kF32) process_row_sub<kF32>(D, r0 + i, srow, T, rv);
                else process_row_sub<kBF16>(D, r0 + i, srow, T, rv);
            }
        } else {
            for (int i = lslot; i < nr; i += slots, ++seq) {
                uint32_t row = stage + (uint32_t)i * row_bytes;
                if constexpr (kColScale) {
                    scale_row(row, (int)D.cols, D.dtype, D.colscale, T.tl, lpr);
                    if (T.G > 1) T.team_sync();
                    else __syncwarp();
                    row = launder_row(row);
                }
                uint32_t* bc = bcast + T.slot * kBcastWords;
                uint32_t* hs = hist + T.slot * 256;
                if (D.dtype == kF32) process_row_team<kF32>(D, r0 + i, row, T, lists, bc, hs, seq);
                else process_row_team<kBF16>(D, r0 + i, row, T, lists, bc, hs, seq);
            }
        }
        // Release the stage: the acquire-release increment orders this warp's
        // reads of the stage before the refill that the last reader starts.
        __syncwarp();
        if (lane == 0) {
            const uint32_t before = atom_add_acq_rel(smem_u32(&done[s]), 1u);
            if ((before + 1u) % (uint32_t)wpt == 0u && t + (int64_t)S * gridDim.x < ntiles && !aborted) {
                issue_tile(P, it + S, di_issue, smem_base, SB, S, full_bar(s, k + 1));
                atomicMax(&last_fill[s], k + 1);
            }
        }
    }
    // No copy may still be landing when the block exits.  Only the latest
    // fill of a stage can be incomplete: a later fill is issued only by a warp
    // whose own wait saw the earlier one complete.  The last warp to leave
    // the loop (no fill is issued after that) waits, bounded, for the latest
    // fill of every stage; instant unless a wait gave up.  (No CTA-wide
    // barrier here: a tile-team that is done must not meet the other team's
    // shape-change barrier, which uses barrier 0 with a different count.)
    __syncwarp();
    if (lane == 0 && atom_add_acq_rel(smem_u32(exited), 1u) == (uint32_t)kTmaConsumerWarps - 1u)
        for (int st = 0; st < S; ++st) {
            const int f = atomicAdd(&last_fill[st], 0);
            if (f >= 0) (void)mbar_wait(full_bar(st, f), full_parity(f), P.wait_ns);
        }
}

}  // namespace gq
