// gq_kernels.cuh -- libgq kernels for sm_100a.
//
//  rowquant_kernel<TW>   per-row clip select (register top-m or in-team radix
//                        select) fused with scale, quantize, dequant, code and
//                        int6/int8 pack output; per-tensor groups read their
//                        clip from the workspace.  A team of TW warps owns a
//                        row; the row is read twice (select, then quantize;
//                        the second read is served from L2).
//  ptsel_kernel<PASS>    per-tensor radix select, three histogram passes
//                        (11 + 11 + 9 bits of |w|); the last block of each
//                        tensor picks the bucket (ticket counter, no spin).
//  ste_kernel            straight-through backward: copy or accumulate.
//  dequant_kernel        dequant on load from packed codes + binary16 scales.
//  passthrough_kernel    binary16 round-to-nearest-even of small tensors.
#pragma once

#include "gq_device.cuh"

namespace gq {

constexpr int kMaxDesc = 96;
constexpr int kBlockWarps = 8;
constexpr int kBlockThreads = kBlockWarps * 32;
constexpr int kTopMax = 8;           // m above this uses radix select

// One tensor of a row-kernel launch (device view of a gq_tensor).
struct RowDesc {
    const void* w;
    void* dq;
    int8_t* codes;
    uint8_t* packed;
    uint16_t* sf16;
    float* sf32;
    float* clip_out;
    const uint32_t* clip_in;   // per-tensor group: selected key in workspace
    int32_t* status;
    int64_t rows, cols, ld, prb;
    int64_t items;             // rows handled (1 when only scalar outputs)
    int32_t m;                 // rank from the top of the clip (per row)
    int32_t qmax;
    int32_t dtype;
    int32_t qbits;
    int32_t export_mode;
    int32_t flags;             // kVec* bits
    int32_t tile_rows;         // pipelined kernel: rows per shared-memory tile
    int32_t lanes_per_row;     // pipelined kernel: threads per row (8 .. 512)
    int32_t out_mode;          // pipelined kernel: output configuration, -1 generic
    int32_t pad2;
};

constexpr int32_t kVecIn = 1;       // rows of w are 16-byte (f32) / 8-byte (bf16) aligned
constexpr int32_t kVecDq = 2;       // rows of dq likewise
constexpr int32_t kVecCodes = 4;    // rows of codes 4-byte aligned
constexpr int32_t kVecPacked = 8;   // rows of packed 4-byte aligned
constexpr int32_t kPerTensor = 16;
constexpr int32_t kElemOut = 32;    // dq, codes or packed requested

struct RowParams {
    int32_t ndesc;
    int32_t pad;
    int64_t start[kMaxDesc + 1];   // prefix sums of items
    RowDesc d[kMaxDesc];
};

__device__ __forceinline__ int find_desc(const int64_t* start, int n, int64_t item) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (start[mid] <= item) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Four consecutive elements of a row (elements past n read as 0).
__device__ __forceinline__ void load_quad(const char* rowp, int dtype, int64_t e0, int64_t n,
                                          bool vec, float v[4]) {
    if (vec && e0 + 3 < n) {
        if (dtype == kF32) {
            float4 x = *reinterpret_cast<const float4*>(rowp + e0 * 4);
            v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
        } else {
            uint2 x = *reinterpret_cast<const uint2*>(rowp + e0 * 2);
            v[0] = bf16_bits_to_float(x.x & 0xFFFFu);
            v[1] = bf16_bits_to_float(x.x >> 16);
            v[2] = bf16_bits_to_float(x.y & 0xFFFFu);
            v[3] = bf16_bits_to_float(x.y >> 16);
        }
        return;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int64_t e = e0 + i;
        float x = 0.0f;
        if (e < n) {
            if (dtype == kF32)
                x = reinterpret_cast<const float*>(rowp)[e];
            else
                x = bf16_bits_to_float(reinterpret_cast<const uint16_t*>(rowp)[e]);
        }
        v[i] = x;
    }
}

// ------------------------------------------------------- clip selection --

// m-th largest key of the row (.x) and the largest key (.y) through a
// register top-M list per lane.
template <int TW, int M>
__device__ uint2 select_topm(const char* rowp, int dtype, int64_t n, bool vec, int m,
                                int tw_warp, int lane, int team,
                                uint32_t (*s_lists)[kTopMax]) {
    TopM<M> T;
    T.init();
    const int64_t nq = (n + 3) >> 2;
    for (int64_t jb = (int64_t)tw_warp * 32; jb < nq; jb += TW * 32) {
        int64_t j = jb + lane;
        if (j < nq) {
            float v[4];
            load_quad(rowp, dtype, 4 * j, n, vec, v);
#pragma unroll
            for (int i = 0; i < 4; ++i) T.insert(abs_key(v[i]));
        }
    }
    T.warp_reduce();
    if constexpr (TW == 1) {
        return make_uint2(T.v[m - 1], T.v[0]);
    } else {
        const int wslot = team * TW + tw_warp;
        if (lane == 0) {
#pragma unroll
            for (int i = 0; i < M; ++i) s_lists[wslot][i] = T.v[i];
        }
        team_sync<TW, kBlockWarps>(team);
        TopM<M> R;
        R.init();
        for (int w = 0; w < TW; ++w) R.merge(s_lists[team * TW + w]);
        team_sync<TW, kBlockWarps>(team);   // lists may be rewritten next row
        return make_uint2(R.v[m - 1], R.v[0]);
    }
}

// m-th largest key through an MSB-first radix select (8+8+8+7 bits of the
// 31-bit key) with a shared histogram per team.  Sets *nonfinite when a key
// has an all-ones exponent.
template <int TW>
__device__ uint32_t select_radix(const char* rowp, int dtype, int64_t n, bool vec, int64_t m,
                                 int tw_warp, int lane, int team, uint32_t* hist,
                                 uint32_t* bcast, bool* nonfinite) {
    const int tt = tw_warp * 32 + lane;
    const int64_t nq = (n + 3) >> 2;
    uint32_t prefix = 0, pmask = 0;
    int64_t rem = m;
    *nonfinite = false;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = pass == 0 ? 23 : pass == 1 ? 15 : pass == 2 ? 7 : 0;
        const uint32_t dmask = pass == 3 ? 0x7Fu : 0xFFu;
        for (int i = tt; i < 256; i += TW * 32) hist[i] = 0u;
        team_sync<TW, kBlockWarps>(team);
        for (int64_t jb = (int64_t)tw_warp * 32; jb < nq; jb += TW * 32) {
            int64_t j = jb + lane;
            if (j < nq) {
                float v[4];
                load_quad(rowp, dtype, 4 * j, n, vec, v);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t key = abs_key(v[i]);
                    if (4 * j + i < n && (key & pmask) == prefix)
                        atomicAdd(&hist[(key >> shift) & dmask], 1u);
                }
            }
        }
        team_sync<TW, kBlockWarps>(team);
        if (tw_warp == 0) {
            // lane l owns bins 255-8l .. 248-8l (descending)
            uint32_t cnt[8];
            uint32_t sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cnt[i] = hist[255 - 8 * lane - i];
                sum += cnt[i];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                uint32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off) incl += o;
            }
            int64_t excl = (int64_t)(incl - sum);
            if (excl < rem && rem <= excl + (int64_t)sum) {
                int64_t acc = excl;
                for (int i = 0; i < 8; ++i) {
                    if (acc + cnt[i] >= rem) {
                        bcast[0] = (uint32_t)(255 - 8 * lane - i);
                        bcast[1] = (uint32_t)(rem - acc);
                        break;
                    }
                    acc += cnt[i];
                }
            }
            if (pass == 0 && lane == 0) bcast[2] = hist[255];
        }
        team_sync<TW, kBlockWarps>(team);
        uint32_t b = bcast[0];
        rem = bcast[1];
        if (pass == 0) *nonfinite = bcast[2] != 0u;
        prefix |= b << shift;
        pmask |= dmask << shift;
        team_sync<TW, kBlockWarps>(team);   // bcast / hist reused next pass
    }
    return prefix;
}

// --------------------------------------------------- quantize + outputs --

template <int TW>
__device__ void quantize_row(const RowDesc& D, int64_t r, const Scale& S, int tw_warp, int lane) {
    const int64_t n = D.cols;
    const int64_t nq = (n + 3) >> 2;
    const int esz = D.dtype == kF32 ? 4 : 2;
    const char* rowp = reinterpret_cast<const char*>(D.w) + r * D.ld * esz;
    char* dqrow = D.dq ? reinterpret_cast<char*>(D.dq) + r * n * esz : nullptr;
    int8_t* crow = D.codes ? D.codes + r * n : nullptr;
    uint8_t* prow = D.packed ? D.packed + r * D.prb : nullptr;
    const bool vin = D.flags & kVecIn, vdq = D.flags & kVecDq;
    const bool vcodes = D.flags & kVecCodes, vpk = D.flags & kVecPacked;
    const bool six = D.qbits == 6;

    for (int64_t jb = (int64_t)tw_warp * 32; jb < nq; jb += TW * 32) {
        const int64_t j = jb + lane;
        const bool valid = j < nq;
        const int64_t e0 = 4 * j;
        const bool full = e0 + 3 < n;
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        if (valid) load_quad(rowp, D.dtype, e0, n, vin, v);
        float b[4];
        int q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            b[i] = quantize_offset(v[i], S);
            q[i] = offset_to_code(b[i]);
        }
        if (valid && dqrow) {
            float d[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) d[i] = offset_to_dq(b[i], S);
            if (D.dtype == kF32) {
                float* o = reinterpret_cast<float*>(dqrow);
                if (vdq && full) {
                    *reinterpret_cast<float4*>(o + e0) = make_float4(d[0], d[1], d[2], d[3]);
                } else {
                    for (int i = 0; i < 4; ++i)
                        if (e0 + i < n) o[e0 + i] = d[i];
                }
            } else {
                uint16_t* o = reinterpret_cast<uint16_t*>(dqrow);
                uint16_t h[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) h[i] = float_to_bf16_bits(d[i]);
                if (vdq && full) {
                    *reinterpret_cast<uint2*>(o + e0) =
                        make_uint2((uint32_t)h[0] | ((uint32_t)h[1] << 16),
                                   (uint32_t)h[2] | ((uint32_t)h[3] << 16));
                } else {
                    for (int i = 0; i < 4; ++i)
                        if (e0 + i < n) o[e0 + i] = h[i];
                }
            }
        }
        const uint32_t bytes4 = (uint32_t)(q[0] & 0xFF) | ((uint32_t)(q[1] & 0xFF) << 8) |
                                ((uint32_t)(q[2] & 0xFF) << 16) | ((uint32_t)(q[3] & 0xFF) << 24);
        if (valid && crow) {
            if (vcodes && full) {
                *reinterpret_cast<uint32_t*>(crow + e0) = bytes4;
            } else {
                for (int i = 0; i < 4; ++i)
                    if (e0 + i < n) crow[e0 + i] = (int8_t)q[i];
            }
        }
        if (prow) {
            if (six) {
                const uint32_t v24 = (uint32_t)(q[0] & 63) | ((uint32_t)(q[1] & 63) << 6) |
                                     ((uint32_t)(q[2] & 63) << 12) | ((uint32_t)(q[3] & 63) << 18);
                const uint32_t nxt = __shfl_down_sync(0xFFFFFFFFu, v24, 1);
                const int sub = lane & 3;
                const int64_t g0 = j - sub;                 // first quad of the 4-lane group
                const bool gfull = vpk && (g0 + 3 < nq);
                if (valid) {
                    if (gfull) {
                        if (sub < 3) {
                            uint32_t word = (v24 >> (8 * sub)) | (nxt << (24 - 8 * sub));
                            *reinterpret_cast<uint32_t*>(prow + 3 * g0 + 4 * sub) = word;
                        }
                    } else {
                        prow[3 * j + 0] = (uint8_t)(v24 & 0xFFu);
                        prow[3 * j + 1] = (uint8_t)((v24 >> 8) & 0xFFu);
                        prow[3 * j + 2] = (uint8_t)((v24 >> 16) & 0xFFu);
                    }
                }
            } else if (valid) {
                if (vpk && full) {
                    *reinterpret_cast<uint32_t*>(prow + e0) = bytes4;
                } else {
                    for (int i = 0; i < 4; ++i)
                        if (e0 + i < n) prow[e0 + i] = (uint8_t)q[i];
                }
            }
        }
    }
}

template <int TW>
__global__ void __launch_bounds__(kBlockThreads)
rowquant_kernel(const __grid_constant__ RowParams P) {
    constexpr int kTeams = kBlockWarps / TW;
    __shared__ uint32_t s_hist[kTeams][256];
    __shared__ uint32_t s_lists[kBlockWarps][kTopMax];
    __shared__ uint32_t s_bcast[kTeams][4];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int team = warp / TW, tw_warp = warp % TW;
    const int64_t total = P.start[P.ndesc];

    for (int64_t item = (int64_t)blockIdx.x * kTeams + team; item < total;
         item += (int64_t)gridDim.x * kTeams) {
        const int di = find_desc(P.start, P.ndesc, item);
        const RowDesc& D = P.d[di];
        const int64_t r = item - P.start[di];
        const int esz = D.dtype == kF32 ? 4 : 2;
        const char* rowp = reinterpret_cast<const char*>(D.w) + r * D.ld * esz;
        const bool vin = D.flags & kVecIn;

        uint32_t ckey;
        bool nonfinite = false;
        if (D.clip_in) {
            ckey = *D.clip_in;
        } else {
            const int m = D.m;
            uint2 sel;
            if (m <= 1)
                sel = select_topm<TW, 1>(rowp, D.dtype, D.cols, vin, 1, tw_warp, lane, team, s_lists);
            else if (m <= 2)
                sel = select_topm<TW, 2>(rowp, D.dtype, D.cols, vin, m, tw_warp, lane, team, s_lists);
            else if (m <= 4)
                sel = select_topm<TW, 4>(rowp, D.dtype, D.cols, vin, m, tw_warp, lane, team, s_lists);
            else if (m <= kTopMax)
                sel = select_topm<TW, 8>(rowp, D.dtype, D.cols, vin, m, tw_warp, lane, team, s_lists);
            else
                sel.x = select_radix<TW>(rowp, D.dtype, D.cols, vin, m, tw_warp, lane, team,
                                         s_hist[team], s_bcast[team], &nonfinite);
            ckey = sel.x;
            if (m <= kTopMax) nonfinite = sel.y >= 0x7F800000u;
        }

        uint16_t hbits;
        bool range;
        const Scale S = make_scale(ckey, D.qmax, D.export_mode != 0, &hbits, &range);
        const bool leader = (tw_warp == 0) && (lane == 0);
        const bool per_tensor = D.flags & kPerTensor;
        if (leader && (!per_tensor || r == 0)) {
            const int64_t g = per_tensor ? 0 : r;
            if (D.clip_out) D.clip_out[g] = S.c;
            if (D.sf32) D.sf32[g] = S.s;
            if (D.sf16) D.sf16[g] = hbits;
            if (D.status) {
                uint32_t st = (nonfinite ? kStatusNonfinite : 0u) | (range ? kStatusRange : 0u);
                if (st) atomicOr(reinterpret_cast<unsigned int*>(D.status), st);
            }
        }
        if (D.flags & kElemOut) quantize_row<TW>(D, r, S, tw_warp, lane);
    }
}

// ------------------------------------------------- per-tensor selection --

struct SelDesc {
    const void* w;
    uint32_t* hist;            // 2048 counters in the workspace
    uint32_t* state;           // [0] prefix [1] remaining [2] ticket [3] key
    int32_t* status;
    int64_t rows, cols, ld;
    int64_t rows_per_item;
    int64_t items;
    int64_t m;
    int32_t dtype;
    int32_t pad;
};

struct SelParams {
    int32_t ndesc;
    int32_t pad;
    int64_t start[kMaxDesc + 1];
    SelDesc d[kMaxDesc];
};

constexpr int kSelBins = 2048;

// PASS 0: digit = key bits 30..20; PASS 1: bits 19..9 among keys whose bits
// 30..20 equal the chosen prefix; PASS 2: bits 8..0 among keys whose bits
// 30..9 match.  One block per item (a block of rows of one tensor).
template <int PASS>
__global__ void __launch_bounds__(kBlockThreads)
ptsel_kernel(const __grid_constant__ SelParams P) {
    __shared__ uint32_t h[kSelBins];
    __shared__ uint32_t s_warp[kBlockWarps];
    __shared__ int s_last;
    const int tid = threadIdx.x;
    const int64_t item = blockIdx.x;
    const int di = find_desc(P.start, P.ndesc, item);
    const SelDesc& D = P.d[di];
    const int64_t it = item - P.start[di];

    for (int i = tid; i < kSelBins; i += kBlockThreads) h[i] = 0u;
    __syncthreads();

    const uint32_t prefix = PASS == 0 ? 0u : __ldcg(&D.state[0]);
    const int64_t r0 = it * D.rows_per_item;
    const int64_t r1 = min(D.rows, r0 + D.rows_per_item);
    const int esz = D.dtype == kF32 ? 4 : 2;
    bool bad = false;
    for (int64_t r = r0; r < r1; ++r) {
        const char* rowp = reinterpret_cast<const char*>(D.w) + r * D.ld * esz;
        for (int64_t c = tid; c < D.cols; c += kBlockThreads) {
            float x = D.dtype == kF32 ? reinterpret_cast<const float*>(rowp)[c]
                                      : bf16_bits_to_float(reinterpret_cast<const uint16_t*>(rowp)[c]);
            uint32_t key = abs_key(x);
            if (PASS == 0) {
                bad |= key >= 0x7F800000u;
                atomicAdd(&h[key >> 20], 1u);
            } else if (PASS == 1) {
                if ((key >> 20) == prefix) atomicAdd(&h[(key >> 9) & 0x7FFu], 1u);
            } else {
                if ((key >> 9) == prefix) atomicAdd(&h[key & 0x1FFu], 1u);
            }
        }
    }
    if (PASS == 0) {
        bad = __syncthreads_or(bad);
        if (bad && tid == 0 && D.status) atomicOr(reinterpret_cast<unsigned int*>(D.status), kStatusNonfinite);
    } else {
        __syncthreads();
    }
    for (int i = tid; i < kSelBins; i += kBlockThreads)
        if (h[i]) atomicAdd(&D.hist[i], h[i]);
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        unsigned int t = atomicAdd(reinterpret_cast<unsigned int*>(&D.state[2]), 1u);
        s_last = (t == (unsigned int)(D.items - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // Last block of this tensor: pick the bucket holding the rem-th largest.
    const int64_t rem = PASS == 0 ? D.m : (int64_t)__ldcg(&D.state[1]);
    const int nb = PASS == 2 ? 512 : kSelBins;
    const int per = nb / kBlockThreads;          // 8 or 2 bins per thread
    uint32_t sum = 0;
    for (int i = 0; i < per; ++i) sum += __ldcg(&D.hist[nb - 1 - per * tid - i]);
    // block-wide inclusive scan of sum (thread order = descending bins)
    const int warp = tid >> 5, lane = tid & 31;
    uint32_t incl = sum;
    for (int off = 1; off < 32; off <<= 1) {
        uint32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    uint32_t wbase = 0;
    for (int w = 0; w < warp; ++w) wbase += s_warp[w];
    const int64_t excl = (int64_t)wbase + (int64_t)(incl - sum);
    if (excl < rem && rem <= excl + (int64_t)sum) {
        int64_t acc = excl;
        for (int i = 0; i < per; ++i) {
            const int bin = nb - 1 - per * tid - i;
            const uint32_t c = __ldcg(&D.hist[bin]);
            if (acc + c >= rem) {
                uint32_t np = PASS == 0 ? (uint32_t)bin
                            : PASS == 1 ? ((prefix << 11) | (uint32_t)bin)
                                        : ((prefix << 9) | (uint32_t)bin);
                D.state[0] = np;
                D.state[1] = (uint32_t)(rem - acc);
                if (PASS == 2) D.state[3] = np;
                break;
            }
            acc += c;
        }
    }
    __syncthreads();
    for (int i = tid; i < kSelBins; i += kBlockThreads) D.hist[i] = 0u;
    if (tid == 0) D.state[2] = 0u;
}

// ------------------------------------------------------------ elementwise --

// g_w = g_out (copy) or g_w += g_out; dense, n16 16-byte vectors then a tail.
__global__ void __launch_bounds__(kBlockThreads)
ste_kernel(const void* __restrict__ g_out, void* __restrict__ g_w, int dtype, int64_t numel,
           int accumulate, int vec) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int per = dtype == kF32 ? 4 : 8;       // elements per 16 bytes
    int64_t nvec = vec ? numel / per : 0;
    const uint4* src = reinterpret_cast<const uint4*>(g_out);
    uint4* dst = reinterpret_cast<uint4*>(g_w);
    for (int64_t i = tid; i < nvec; i += stride) {
        uint4 a = src[i];
        if (accumulate) {
            uint4 b = dst[i];
            if (dtype == kF32) {
                a.x = __float_as_uint(__fadd_rn(__uint_as_float(b.x), __uint_as_float(a.x)));
                a.y = __float_as_uint(__fadd_rn(__uint_as_float(b.y), __uint_as_float(a.y)));
                a.z = __float_as_uint(__fadd_rn(__uint_as_float(b.z), __uint_as_float(a.z)));
                a.w = __float_as_uint(__fadd_rn(__uint_as_float(b.w), __uint_as_float(a.w)));
            } else {
                uint32_t* pa = &a.x;
                const uint32_t* pb = &b.x;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float lo = __fadd_rn(bf16_bits_to_float(pb[k] & 0xFFFFu), bf16_bits_to_float(pa[k] & 0xFFFFu));
                    float hi = __fadd_rn(bf16_bits_to_float(pb[k] >> 16), bf16_bits_to_float(pa[k] >> 16));
                    pa[k] = (uint32_t)float_to_bf16_bits(lo) | ((uint32_t)float_to_bf16_bits(hi) << 16);
                }
            }
        }
        dst[i] = a;
    }
    for (int64_t e = nvec * per + tid; e < numel; e += stride) {
        if (dtype == kF32) {
            float a = reinterpret_cast<const float*>(g_out)[e];
            float* o = reinterpret_cast<float*>(g_w) + e;
            *o = accumulate ? __fadd_rn(*o, a) : a;
        } else {
            uint16_t a = reinterpret_cast<const uint16_t*>(g_out)[e];
            uint16_t* o = reinterpret_cast<uint16_t*>(g_w) + e;
            *o = accumulate ? float_to_bf16_bits(__fadd_rn(bf16_bits_to_float(*o), bf16_bits_to_float(a))) : a;
        }
    }
}

// out[r, c] = (float)q * (float)h[r]; one thread per quad of codes.
__global__ void __launch_bounds__(kBlockThreads)
dequant_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ sf16, int qbits,
               int per_tensor, int64_t rows, int64_t cols, int64_t prb, void* __restrict__ out,
               int out_dtype, int vec_out) {
    const int64_t nq = (cols + 3) >> 2;
    const int64_t total = rows * nq;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += stride) {
        const int64_t r = t / nq, j = t - r * nq;
        const uint16_t hb = sf16[per_tensor ? 0 : r];
        const float s = __half2float(*reinterpret_cast<const __half*>(&hb));
        const uint8_t* prow = packed + r * prb;
        int q[4];
        if (qbits == 6) {
            uint32_t v = (uint32_t)prow[3 * j] | ((uint32_t)prow[3 * j + 1] << 8) |
                         ((uint32_t)prow[3 * j + 2] << 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int u = (int)((v >> (6 * i)) & 63u);
                q[i] = u >= 32 ? u - 64 : u;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) q[i] = (4 * j + i < cols) ? (int)(int8_t)prow[4 * j + i] : 0;
        }
        const int64_t e0 = 4 * j;
        const bool full = e0 + 3 < cols;
        float d[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) d[i] = __fmul_rn((float)q[i], s);
        if (out_dtype == kF32) {
            float* o = reinterpret_cast<float*>(out) + r * cols;
            if (vec_out && full)
                *reinterpret_cast<float4*>(o + e0) = make_float4(d[0], d[1], d[2], d[3]);
            else
                for (int i = 0; i < 4; ++i)
                    if (e0 + i < cols) o[e0 + i] = d[i];
        } else {
            uint16_t* o = reinterpret_cast<uint16_t*>(out) + r * cols;
            for (int i = 0; i < 4; ++i)
                if (e0 + i < cols) o[e0 + i] = float_to_bf16_bits(d[i]);
        }
    }
}

// Binary16 passthrough of a batch of small tensors: out[r, c] = binary16(w[r, c]).
struct PassDesc {
    const void* w;
    uint16_t* out;
    int64_t rows, cols, ld;
    int32_t dtype;
    int32_t pad;
};

struct PassParams {
    int32_t ndesc;
    int32_t pad;
    int64_t start[kMaxDesc + 1];   // prefix sums of 1024-element chunks
    PassDesc d[kMaxDesc];
};

constexpr int kPassChunk = 1024;

__global__ void __launch_bounds__(kBlockThreads)
passthrough_kernel(const __grid_constant__ PassParams P) {
    const int64_t total = P.start[P.ndesc];
    for (int64_t item = blockIdx.x; item < total; item += gridDim.x) {
        const int di = find_desc(P.start, P.ndesc, item);
        const PassDesc& D = P.d[di];
        const int64_t numel = D.rows * D.cols;
        const int64_t e_begin = (item - P.start[di]) * kPassChunk;
        const int64_t e_end = min(numel, e_begin + kPassChunk);
        for (int64_t e = e_begin + threadIdx.x; e < e_end; e += blockDim.x) {
            const int64_t r = e / D.cols, c = e - r * D.cols;
            float x = D.dtype == kF32
                          ? reinterpret_cast<const float*>(D.w)[r * D.ld + c]
                          : bf16_bits_to_float(reinterpret_cast<const uint16_t*>(D.w)[r * D.ld + c]);
            __half h = __float2half_rn(x);
            D.out[e] = *reinterpret_cast<uint16_t*>(&h);
        }
    }
}

}  // namespace gq
