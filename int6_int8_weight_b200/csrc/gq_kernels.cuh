// gq_kernels.cuh -- libgq kernels for sm_100a.
//
//  rowquant_kernel<TW>   per-row clip select (register top-m or in-team radix
//                        select) fused with scale, quantize, dequant, code and
//                        int6/int8 pack output; per-tensor groups read their
//                        clip from the workspace.  A team of TW warps owns a
//                        row; the row is read twice (select, then quantize;
//                        the second read is served from L2).
// (per-tensor selection, STE backward, dequant and passthrough kernels are
// in gq_aux_kernels.cuh)
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
    int32_t avg_kind;          // kAvg*: running average of the w_hat snapshots
    float* avg;                // binary32 [rows, cols] averages (dense), or null
    float avg_t;               // mean: RN(1 / (n + 1)); EMA: decay
    float avg_c;               // EMA: RN(1 - decay)
    const float* colscale;     // AWQ: binary32 [cols] column scales, or null
};

constexpr int32_t kVecIn = 1;       // rows of w are 16-byte (f32) / 8-byte (bf16) aligned
constexpr int32_t kVecDq = 2;       // rows of dq likewise
constexpr int32_t kVecCodes = 4;    // rows of codes 4-byte aligned
constexpr int32_t kVecPacked = 8;   // rows of packed 4-byte aligned
constexpr int32_t kPerTensor = 16;
constexpr int32_t kElemOut = 32;    // dq, codes, packed or an average requested
constexpr int32_t kVecAvg = 64;     // rows of the average 16-byte aligned
constexpr int32_t kVecCol = 128;    // the column scales 16-byte aligned

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

// Four consecutive elements of a row (elements past n read as 0).  With
// column scales cs (AWQ), element e is the column-scaled weight
// RN_dtype(w[e] * cs[e]): one binary32 multiply, rounded to nearest even
// bf16 for a bf16 weight (the weight rescaled in its own dtype).
__device__ __forceinline__ float col_scaled(float x, float t, int dtype) {
    const float y = __fmul_rn(x, t);
    return dtype == kF32 ? y : bf16_bits_to_float(float_to_bf16_bits(y));
}

__device__ __forceinline__ void load_quad(const char* rowp, int dtype, int64_t e0, int64_t n,
                                          bool vec, float v[4], const float* cs = nullptr,
                                          bool vcs = false) {
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
    } else {
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
    if (cs) {
        if (vcs && e0 + 3 < n) {
            const float4 t = __ldg(reinterpret_cast<const float4*>(cs + e0));
            v[0] = col_scaled(v[0], t.x, dtype);
            v[1] = col_scaled(v[1], t.y, dtype);
            v[2] = col_scaled(v[2], t.z, dtype);
            v[3] = col_scaled(v[3], t.w, dtype);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (e0 + i < n) v[i] = col_scaled(v[i], __ldg(cs + e0 + i), dtype);
        }
    }
}

// ------------------------------------------------------- clip selection --

// m-th largest key of the row (.x) and the largest key (.y) through a
// register top-M list per lane.
template <int TW, int M>
__device__ uint2 select_topm(const char* rowp, int dtype, int64_t n, bool vec, int m,
                                int tw_warp, int lane, int team,
                                uint32_t (*s_lists)[kTopMax], const float* cs, bool vcs) {
    TopM<M> T;
    T.init();
    const int64_t nq = (n + 3) >> 2;
    for (int64_t jb = (int64_t)tw_warp * 32; jb < nq; jb += TW * 32) {
        int64_t j = jb + lane;
        if (j < nq) {
            float v[4];
            load_quad(rowp, dtype, 4 * j, n, vec, v, cs, vcs);
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
                                 uint32_t* bcast, bool* nonfinite, const float* cs, bool vcs) {
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
                load_quad(rowp, dtype, 4 * j, n, vec, v, cs, vcs);
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
        if (valid) load_quad(rowp, D.dtype, e0, n, vin, v, D.colscale, (D.flags & kVecCol) != 0);
        float b[4];
        int q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            b[i] = quantize_offset(v[i], S);
            q[i] = offset_to_code(b[i]);
        }
        if (valid && D.avg) {
            // the snapshot as the model holds it: bf16 w_hat widened
            float* arow = D.avg + r * n;
            const AvgOp A{arow, D.avg_t, D.avg_c, D.avg_kind};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (e0 + i < n) {
                    float x = offset_to_dq(b[i], S);
                    if (D.dtype != kF32) x = bf16_bits_to_float(float_to_bf16_bits(x));
                    arow[e0 + i] = avg_update(arow[e0 + i], x, A);
                }
            }
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
        const float* cs = D.colscale;
        const bool vcs = (D.flags & kVecCol) != 0;

        uint32_t ckey;
        bool nonfinite = false;
        if (D.clip_in) {
            ckey = *D.clip_in;
        } else {
            const int m = D.m;
            uint2 sel;
            if (m <= 1)
                sel = select_topm<TW, 1>(rowp, D.dtype, D.cols, vin, 1, tw_warp, lane, team, s_lists, cs, vcs);
            else if (m <= 2)
                sel = select_topm<TW, 2>(rowp, D.dtype, D.cols, vin, m, tw_warp, lane, team, s_lists, cs, vcs);
            else if (m <= 4)
                sel = select_topm<TW, 4>(rowp, D.dtype, D.cols, vin, m, tw_warp, lane, team, s_lists, cs, vcs);
            else if (m <= kTopMax)
                sel = select_topm<TW, 8>(rowp, D.dtype, D.cols, vin, m, tw_warp, lane, team, s_lists, cs, vcs);
            else
                sel.x = select_radix<TW>(rowp, D.dtype, D.cols, vin, m, tw_warp, lane, team,
                                         s_hist[team], s_bcast[team], &nonfinite, cs, vcs);
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

}  // namespace gq
