// gq_api.cu -- the libgq C ABI (include/gq.h): argument checks, launch
// planning and kernel launches.  Host code only; kernels are in
// gq_kernels.cuh.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstddef>
#include <cstring>
#include <string>
#include <vector>

#include "gq.h"
#include <cudaTypedefs.h>

#include "gq_aux_kernels.cuh"
#include "gq_gemm.cuh"
#include "gq_gemm_decode.cuh"
#include "gq_gptq.cuh"
#include "gq_kernels.cuh"
#include "gq_rowquant_tma.cuh"

namespace {

using namespace gq;

constexpr size_t kWsSlot = 8448;      // 2048 x u32 histogram + 16 x u32 state, 256-aligned
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    int v = g_sm_count[dev].load(std::memory_order_relaxed);
    if (v <= 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
            v = 148;
        g_sm_count[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int64_t k_from_p(int64_t n, double p) {
    double prod = p * (double)n;
    double up = std::ceil(prod);
    int64_t k = (int64_t)up;
    if (k < 1) k = 1;
    if (k > n) k = n;
    return k;
}

int64_t packed_row_bytes(int64_t cols, int qbits) {
    if (cols < 0) return -1;
    if (qbits == 6) return 3 * ((cols + 3) / 4);
    if (qbits == 8) return cols;
    if (qbits == 16) return 2 * cols;
    return -1;
}

enum class Op { Select, FakeQuant, Export, Average };

// Validate one descriptor for an operation.  Returns GQ_OK or an error.
// The running average that goes with a tensor of gq_fakequant_average.
gq_status check_avg(const gq_tensor& t, const gq_avg& a) {
    if (a.kind != GQ_AVG_MEAN && a.kind != GQ_AVG_EMA) return GQ_ERR_INVALID_ARG;
    if (a.kind == GQ_AVG_MEAN && (a.count < 0 || a.count >= (int64_t)1 << 24)) return GQ_ERR_INVALID_ARG;
    if (a.kind == GQ_AVG_EMA && !(a.decay >= 0.0f && a.decay <= 1.0f)) return GQ_ERR_INVALID_ARG;
    if (t.rows == 0 || t.cols == 0) return GQ_OK;
    if (!a.avg) return GQ_ERR_INVALID_ARG;
    if (!aligned(a.avg, 4)) return GQ_ERR_MISALIGNED;
    return GQ_OK;
}

static_assert(sizeof(gq_tensor) == 112 && offsetof(gq_tensor, col_scale) == 104,
              "gq_tensor layout is part of the ABI (the Python binding mirrors it)");

gq_status check_tensor(const gq_tensor& t, Op op, bool f16_mode) {
    if (t.reserved != 0) return GQ_ERR_INVALID_ARG;
    if (t.dtype != GQ_F32 && t.dtype != GQ_BF16) return GQ_ERR_INVALID_ARG;
    if (t.gran != GQ_PER_ROW && t.gran != GQ_PER_TENSOR) return GQ_ERR_INVALID_ARG;
    const bool pass16 = t.qbits == 16;
    if (!(t.qbits == 6 || t.qbits == 8 || (pass16 && op == Op::Export))) return GQ_ERR_INVALID_ARG;
    if (t.rows < 0 || t.cols < 0 || t.ld < t.cols) return GQ_ERR_INVALID_ARG;
    if (t.cols > (int64_t)INT32_MAX) return GQ_ERR_UNSUPPORTED;
    if (!pass16 && !(t.p > 0.0 && t.p <= 1.0)) return GQ_ERR_INVALID_ARG;
    // AWQ column scales: per-row groups of the quantizing calls only
    if (t.col_scale && (pass16 || t.gran != GQ_PER_ROW)) return GQ_ERR_UNSUPPORTED;
    const int64_t esz = t.dtype == GQ_F32 ? 4 : 2;
    if (t.rows > 0 && t.ld > 0 && t.rows > INT64_MAX / 16 / t.ld) return GQ_ERR_INVALID_ARG;
    if (t.rows > 0 && t.cols > 0 && t.rows > INT64_MAX / 16 / t.cols) return GQ_ERR_INVALID_ARG;
    if (t.rows == 0 || t.cols == 0) return GQ_OK;   // empty: nothing read or written
    if (!t.w) return GQ_ERR_INVALID_ARG;
    if (!aligned(t.w, esz)) return GQ_ERR_MISALIGNED;
    if (t.dq && !aligned(t.dq, esz)) return GQ_ERR_MISALIGNED;
    if (t.scale_f16 && !aligned(t.scale_f16, 2)) return GQ_ERR_MISALIGNED;
    if (t.scale_f32 && !aligned(t.scale_f32, 4)) return GQ_ERR_MISALIGNED;
    if (t.clip && !aligned(t.clip, 4)) return GQ_ERR_MISALIGNED;
    if (t.col_scale && !aligned(t.col_scale, 4)) return GQ_ERR_MISALIGNED;
    switch (op) {
        case Op::Select:
            if (!t.clip) return GQ_ERR_INVALID_ARG;
            if (t.dq || t.codes || t.packed || t.scale_f16 || t.scale_f32) return GQ_ERR_INVALID_ARG;
            break;
        case Op::FakeQuant:
            if (!t.dq || t.packed) return GQ_ERR_INVALID_ARG;
            if (t.scale_f16 && !f16_mode) return GQ_ERR_INVALID_ARG;
            break;
        case Op::Average:
            if (t.codes || t.packed) return GQ_ERR_INVALID_ARG;
            if (t.scale_f16 && !f16_mode) return GQ_ERR_INVALID_ARG;
            break;
        case Op::Export:
            if (pass16) {
                if (!t.packed || t.dq || t.codes || t.scale_f16 || t.scale_f32 || t.clip)
                    return GQ_ERR_INVALID_ARG;
                if (!aligned(t.packed, 2)) return GQ_ERR_MISALIGNED;
            } else if (!t.packed || !t.scale_f16) {
                return GQ_ERR_INVALID_ARG;
            }
            break;
    }
    return GQ_OK;
}

bool needs_workspace(const gq_tensor& t) {
    return t.qbits != 16 && t.gran == GQ_PER_TENSOR && t.rows > 0 && t.cols > 0;
}

// A per-tensor group's workspace slot: the histogram and state (kWsSlot),
// then, unless the caller has no room for it, kSelCand candidate keys.
constexpr int32_t kSelCand = 4096;
constexpr size_t kCandBytes = (size_t)kSelCand * 4;
size_t slot_bytes(bool cand) { return kWsSlot + (cand ? kCandBytes : 0); }

size_t workspace_size(const gq_tensor* t, int n, bool cand = true) {
    size_t slots = 0;
    for (int i = 0; i < n; ++i)
        if (needs_workspace(t[i])) ++slots;
    return slots * slot_bytes(cand);
}

thread_local int g_last_cuda_error = 0;

// GQ_OK, or GQ_ERR_CUDA after recording the CUDA error for gq_last_cuda_error.
gq_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return GQ_OK;
    g_last_cuda_error = (int)e;
    return GQ_ERR_CUDA;
}

gq_status launch_status() { return cuda_status(cudaGetLastError()); }

// Per-tensor radix select for every per-tensor descriptor (three passes).
gq_status run_per_tensor_select(const std::vector<SelDesc>& sel, cudaStream_t stream) {
    for (size_t base = 0; base < sel.size(); base += kMaxDesc) {
        SelParams P;
        std::memset(&P, 0, sizeof(P));
        const int nd = (int)std::min<size_t>(kMaxDesc, sel.size() - base);
        P.ndesc = nd;
        int64_t acc = 0;
        for (int i = 0; i < nd; ++i) {
            P.start[i] = acc;
            P.d[i] = sel[base + i];
            acc += P.d[i].items;
        }
        P.start[nd] = acc;
        if (acc == 0) continue;
        if (acc > INT32_MAX) return GQ_ERR_UNSUPPORTED;
        ptsel_kernel<0><<<(unsigned)acc, kBlockThreads, 0, stream>>>(P);
        ptsel_kernel<1><<<(unsigned)acc, kBlockThreads, 0, stream>>>(P);
        ptsel_kernel<2><<<(unsigned)acc, kBlockThreads, 0, stream>>>(P);
        if (launch_status() != GQ_OK) return GQ_ERR_CUDA;
    }
    return GQ_OK;
}

template <int TW>
gq_status run_rows(const std::vector<RowDesc>& rows, cudaStream_t stream) {
    constexpr int kTeams = kBlockWarps / TW;
    const int64_t max_blocks = (int64_t)sm_count() * (2048 / kBlockThreads);
    for (size_t base = 0; base < rows.size(); base += kMaxDesc) {
        RowParams P;
        std::memset(&P, 0, sizeof(P));
        const int nd = (int)std::min<size_t>(kMaxDesc, rows.size() - base);
        P.ndesc = nd;
        int64_t acc = 0;
        for (int i = 0; i < nd; ++i) {
            P.start[i] = acc;
            P.d[i] = rows[base + i];
            acc += P.d[i].items;
        }
        P.start[nd] = acc;
        if (acc == 0) continue;
        const int64_t blocks = std::min<int64_t>(max_blocks, (acc + kTeams - 1) / kTeams);
        rowquant_kernel<TW><<<(unsigned)blocks, kBlockThreads, 0, stream>>>(P);
        if (launch_status() != GQ_OK) return GQ_ERR_CUDA;
    }
    return GQ_OK;
}

// Test hook of the bounded waits (gq_test_arm_wait_expiry): armed per host
// thread, consumed by the next launch of the pipelined row kernel.
thread_local int64_t g_test_poison_tile = -1;
thread_local uint64_t g_test_wait_ns = 0;

// Pipelined launch over the descriptors whose rows can be bulk-copied.
constexpr int kTmaStageBytes = 68 * 1024;
constexpr int kTmaMaxRowBytes = 96 * 1024;
std::atomic<int> g_tma_smem_set[2][kMaxDevices];

bool tma_eligible(const gq_tensor& T, int32_t flags) {
    const int64_t esz = T.dtype == GQ_F32 ? 4 : 2;
    const int64_t row_bytes = T.cols * esz;
    return (flags & kElemOut) && aligned(T.w, 16) && ((T.ld * esz) % 16) == 0 &&
           (row_bytes % 16) == 0 && row_bytes <= kTmaMaxRowBytes;
}

// Output configuration of the branch-free loops, or kOutGeneric.
int32_t tma_out_mode(const RowDesc& D) {
    int32_t mode = 0;
    if (D.avg) {
        if (!(D.flags & kVecAvg)) return kOutGeneric;
        mode |= kOutAvg;
    }
    if (D.dq) {
        if (!(D.flags & kVecDq)) return kOutGeneric;
        mode |= kOutDq;
    }
    if (D.codes) {
        if (!(D.flags & kVecCodes)) return kOutGeneric;
        mode |= kOutCodes;
    }
    if (D.packed) {
        if (!(D.flags & kVecPacked)) return kOutGeneric;
        if (D.qbits == 6) {
            if (D.cols % 16 != 0) return kOutGeneric;   // partial 4-code groups
            mode |= kOutSix;
        }
        mode |= kOutPacked;
    }
    switch (mode) {
        case kOutDq | kOutPacked | kOutSix:
        case kOutDq | kOutPacked:
        case kOutDq:
        case kOutPacked | kOutSix:
        case kOutPacked:
        case kOutDq | kOutCodes | kOutPacked | kOutSix:
        case kOutDq | kOutCodes:
        case kOutAvg:
        case kOutDq | kOutAvg:
            return mode;
        default:
            return kOutGeneric;
    }
}

template <bool kColScale>
gq_status run_rows_tma_impl(std::vector<RowDesc>& rows, cudaStream_t stream) {
    if (rows.empty()) return GQ_OK;
    int64_t max_row = 0;
    for (const RowDesc& D : rows) max_row = std::max<int64_t>(max_row, D.cols * (D.dtype == kF32 ? 4 : 2));
    const int sb = max_row <= kTmaStageBytes ? kTmaStageBytes : (int)((max_row + 15) / 16 * 16);
    const int nstages = max_row <= kTmaStageBytes ? 3 : 2;
    // two tile-teams of 8 warps take alternate tiles when a third stage is
    // left for prefetching; a row then needs half as many threads
    const int teams = nstages == 3 ? 2 : 1;
    const int team_threads = kTmaConsumers / teams;
    for (RowDesc& D : rows) {
        const int64_t row_bytes = D.cols * (D.dtype == kF32 ? 4 : 2);
        const int64_t rmax = sb / row_bytes;
        // radix selection (m > 8, per row) runs on whole warps
        const bool whole_warps = !D.clip_in && D.m > kTopMax;
        // Narrow rows start at 4 threads per row, so fewer threads repeat each
        // row's select and scale set-up, unless the row pitch is a multiple of
        // 128 bytes: then every staged row starts on the same shared-memory
        // bank, and 8 threads per row keep a warp's loads at 4 rows per bank
        // instead of 8.  (bf16 rows: 528 columns take 4 threads, 512 take 8.)
        int lpr = row_bytes % 128 != 0 ? 4 : 8;
        while (lpr < team_threads && (team_threads / lpr > rmax || (whole_warps && lpr < 32))) lpr *= 2;
        const int64_t slots = team_threads / lpr;
        D.tile_rows = (int32_t)(rmax / slots * slots);
        D.lanes_per_row = lpr;
        D.out_mode = tma_out_mode(D);
        D.items = (D.rows + D.tile_rows - 1) / D.tile_rows;
    }
    const size_t smem = (size_t)nstages * sb + kTmaExtraBytes;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQ_ERR_CUDA;
    std::atomic<int>& smem_set = g_tma_smem_set[kColScale ? 1 : 0][dev >= 0 && dev < kMaxDevices ? dev : 0];
    if (dev >= 0 && dev < kMaxDevices && smem_set.load() < (int)smem) {
        if (cuda_status(cudaFuncSetAttribute(rowquant_tma_kernel<kColScale>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != GQ_OK)
            return GQ_ERR_CUDA;
        smem_set.store((int)smem);
    }
    for (size_t base = 0; base < rows.size(); base += kMaxDesc) {
        TmaParams P;
        std::memset(&P, 0, sizeof(P));
        const int nd = (int)std::min<size_t>(kMaxDesc, rows.size() - base);
        P.ndesc = nd;
        P.nstages = nstages;
        P.stage_bytes = sb;
        P.teams = teams;
        P.wait_ns = kWaitLimitNs;
        P.poison_tile = -1;
        if (g_test_poison_tile >= 0) {
            P.wait_ns = g_test_wait_ns;
            P.poison_tile = g_test_poison_tile;
            P.poison_bytes = 16;
            g_test_poison_tile = -1;
        }
        int64_t acc = 0;
        for (int i = 0; i < nd; ++i) {
            P.start[i] = acc;
            P.d[i] = rows[base + i];
            acc += P.d[i].items;
        }
        P.start[nd] = acc;
        if (acc == 0) continue;
        const int64_t blocks = std::min<int64_t>(sm_count(), acc);
        rowquant_tma_kernel<kColScale><<<(unsigned)blocks, kTmaThreads, smem, stream>>>(P);
        if (launch_status() != GQ_OK) return GQ_ERR_CUDA;
    }
    return GQ_OK;
}

// Groups with AWQ column scales go to their own launch of the pipelined kernel.
gq_status run_rows_tma(std::vector<RowDesc>& rows, cudaStream_t stream) {
    std::vector<RowDesc> plain, scaled;
    for (const RowDesc& D : rows) (D.colscale ? scaled : plain).push_back(D);
    gq_status st = run_rows_tma_impl<false>(plain, stream);
    if (st != GQ_OK) return st;
    return run_rows_tma_impl<true>(scaled, stream);
}

gq_status run_passthrough(const std::vector<PassDesc>& pd, cudaStream_t stream) {
    for (size_t base = 0; base < pd.size(); base += kMaxDesc) {
        PassParams P;
        std::memset(&P, 0, sizeof(P));
        const int nd = (int)std::min<size_t>(kMaxDesc, pd.size() - base);
        P.ndesc = nd;
        int64_t acc = 0;
        for (int i = 0; i < nd; ++i) {
            P.start[i] = acc;
            P.d[i] = pd[base + i];
            acc += (P.d[i].rows * P.d[i].cols + kPassChunk - 1) / kPassChunk;
        }
        P.start[nd] = acc;
        if (acc == 0) continue;
        const int64_t blocks = std::min<int64_t>((int64_t)sm_count() * 8, acc);
        passthrough_kernel<<<(unsigned)blocks, kBlockThreads, 0, stream>>>(P);
        if (launch_status() != GQ_OK) return GQ_ERR_CUDA;
    }
    return GQ_OK;
}

// The shared driver of gq_row_clip_select, gq_fakequant_fwd and gq_export_pack.
gq_status quantize_batch(const gq_tensor* t, int n, Op op, bool f16_mode, void* ws,
                         size_t ws_bytes, int32_t* d_status, cudaStream_t stream,
                         const gq_avg* avg = nullptr, bool cand = true) {
    if (n < 0 || (n > 0 && !t)) return GQ_ERR_INVALID_ARG;
    if (op == Op::Average && n > 0 && !avg) return GQ_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        gq_status st = check_tensor(t[i], op, f16_mode);
        if (st != GQ_OK) return st;
        if (op == Op::Average && (st = check_avg(t[i], avg[i])) != GQ_OK) return st;
    }
    const size_t need = workspace_size(t, n, cand);
    if (need > 0) {
        if (!ws || ws_bytes < need) return GQ_ERR_WORKSPACE;
        if (!aligned(ws, 256)) return GQ_ERR_MISALIGNED;
    }
    if (d_status && !aligned(d_status, 4)) return GQ_ERR_MISALIGNED;
    if (n == 0) return GQ_OK;

    if (d_status && cuda_status(cudaMemsetAsync(d_status, 0, sizeof(int32_t) * (size_t)n, stream)) != GQ_OK)
        return GQ_ERR_CUDA;
    if (need > 0 && cuda_status(cudaMemsetAsync(ws, 0, need, stream)) != GQ_OK) return GQ_ERR_CUDA;

    std::vector<SelDesc> sel;
    std::vector<RowDesc> rows_w, rows_c;   // warp teams / block teams
    std::vector<RowDesc> rows_tma;         // pipelined through shared memory
    std::vector<PassDesc> pass;
    size_t slot = 0;
    for (int i = 0; i < n; ++i) {
        const gq_tensor& T = t[i];
        if (T.rows == 0 || T.cols == 0) continue;
        const int esz = T.dtype == GQ_F32 ? 4 : 2;
        int32_t* status = d_status ? d_status + i : nullptr;
        if (T.qbits == 16) {
            PassDesc P{};
            P.w = T.w;
            P.out = reinterpret_cast<uint16_t*>(T.packed);
            P.rows = T.rows;
            P.cols = T.cols;
            P.ld = T.ld;
            P.dtype = T.dtype;
            pass.push_back(P);
            continue;
        }
        RowDesc D{};
        D.w = T.w;
        D.dq = T.dq;
        D.codes = T.codes;
        D.packed = T.packed;
        D.sf16 = ((op == Op::FakeQuant || op == Op::Average) && !f16_mode) ? nullptr : T.scale_f16;
        D.sf32 = T.scale_f32;
        D.clip_out = T.clip;
        D.status = status;
        D.rows = T.rows;
        D.cols = T.cols;
        D.ld = T.ld;
        D.prb = packed_row_bytes(T.cols, T.qbits);
        D.qmax = T.qbits == 6 ? 31 : 127;
        D.dtype = T.dtype;
        D.qbits = T.qbits;
        D.export_mode = (op == Op::Export || f16_mode) ? 1 : 0;
        if (op == Op::Average) {
            const gq_avg& A = avg[i];
            D.avg = A.avg;
            if (A.kind == GQ_AVG_MEAN) {
                D.avg_kind = A.count == 0 ? kAvgCopy : kAvgMean;
                D.avg_t = 1.0f / (float)(A.count + 1);      // one binary32 division
            } else {
                D.avg_kind = kAvgEma;
                D.avg_t = A.decay;
                D.avg_c = 1.0f - A.decay;                   // one binary32 subtraction
            }
        }
        D.colscale = T.col_scale;
        const bool elem = T.dq || T.codes || T.packed || D.avg;
        int32_t flags = elem ? kElemOut : 0;
        if (T.col_scale && aligned(T.col_scale, 16)) flags |= kVecCol;
        if (D.avg && aligned(D.avg, 16) && (T.cols % 4) == 0) flags |= kVecAvg;
        const size_t vin = T.dtype == GQ_F32 ? 16 : 8;
        if (aligned(T.w, vin) && ((T.ld * esz) % (int64_t)vin) == 0) flags |= kVecIn;
        if (T.dq && aligned(T.dq, vin) && ((T.cols * esz) % (int64_t)vin) == 0) flags |= kVecDq;
        if (T.codes && aligned(T.codes, 4) && (T.cols % 4) == 0) flags |= kVecCodes;
        if (T.packed && aligned(T.packed, 4) && (D.prb % 4) == 0) flags |= kVecPacked;
        if (T.gran == GQ_PER_TENSOR) {
            flags |= kPerTensor;
            const int64_t numel = T.rows * T.cols;
            uint8_t* base = static_cast<uint8_t*>(ws) + slot * slot_bytes(cand);
            ++slot;
            SelDesc S{};
            S.w = T.w;
            S.hist = reinterpret_cast<uint32_t*>(base);
            S.state = reinterpret_cast<uint32_t*>(base + kSelBins * sizeof(uint32_t));
            S.cand = cand ? reinterpret_cast<uint32_t*>(base + kWsSlot) : nullptr;
            S.cap = cand ? kSelCand : 0;
            S.status = status;
            S.rows = T.rows;
            S.cols = T.cols;
            S.ld = T.ld;
            S.rows_per_item = std::max<int64_t>(1, 65536 / T.cols);
            S.items = (T.rows + S.rows_per_item - 1) / S.rows_per_item;
            S.m = numel - k_from_p(numel, T.p) + 1;
            S.dtype = T.dtype;
            sel.push_back(S);
            D.clip_in = S.state + 3;
            D.m = S.m > 1 ? 2 : 1;     // clip is given; only "some |w| > c" matters
            D.items = elem ? T.rows : 1;
        } else {
            D.m = (int32_t)(T.cols - k_from_p(T.cols, T.p) + 1);
            D.items = T.rows;
        }
        D.flags = flags;
        // column scales read as float4 by the pipelined kernel (else the row kernels)
        if (tma_eligible(T, flags) && (!T.col_scale || (flags & kVecCol)))
            rows_tma.push_back(D);
        else if (T.cols <= 2048)
            rows_w.push_back(D);
        else
            rows_c.push_back(D);
    }

    // the per-tensor clips first (three streaming passes over those tensors),
    // then every row pass
    gq_status st = run_per_tensor_select(sel, stream);
    if (st != GQ_OK) return st;
    st = run_rows_tma(rows_tma, stream);
    if (st != GQ_OK) return st;
    st = run_rows<1>(rows_w, stream);
    if (st != GQ_OK) return st;
    st = run_rows<kBlockWarps>(rows_c, stream);
    if (st != GQ_OK) return st;
    return run_passthrough(pass, stream);
}

// ---------------------------------------------------- dequant-on-load GEMM --

std::atomic<void*> g_encode_tiled{nullptr};
std::atomic<int> g_gemm_smem_set[2][kMaxDevices];
std::atomic<int> g_dec_smem_set[2][kMaxDevices];

// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on the driver library).
PFN_cuTensorMapEncodeTiled encode_tiled() {
    void* f = g_encode_tiled.load(std::memory_order_acquire);
    if (!f) {
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !f)
            return nullptr;
        g_encode_tiled.store(f, std::memory_order_release);
    }
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled>(f);
}

// Scratch of gq_export_pack_noalloc: a fixed device array that every call on
// a device shares, for callers that cannot hand the library any device memory.
constexpr size_t kNoAllocSlots = 64;                       // per-tensor groups per call
constexpr size_t kNoAllocBytes = kNoAllocSlots * kWsSlot;  // 528 KiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of g_noalloc_scratch in the current context.  Host code
// sees only a host-side stand-in for the array, so the address is looked up
// on every call: after a device reset or in another context the module is
// loaded again and an address kept from before would be stale.
gq_status noalloc_scratch(void** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GQ_ERR_CUDA;
    *out = p;
    return GQ_OK;
}

// ------------------------------------------------------------- GPTQ-lite --

constexpr int64_t kGptqMaxCols = 5800;     // residual rows of a block stay in shared memory

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

struct GptqWs {
    float* clip;
    uint8_t* dead;
    GpState* st;
    double* L;
    size_t bytes;
};

GptqWs gptq_layout(void* base, int64_t rows, int64_t cols) {
    GptqWs w{};
    size_t off = 0;
    auto take = [&](size_t b) {
        size_t o = off;
        off += round256(b);
        return o;
    };
    const size_t o_clip = take((size_t)rows * 4), o_dead = take((size_t)cols), o_st = take(sizeof(GpState)),
                 o_L = take((size_t)cols * (size_t)cols * 8);
    unsigned char* b = static_cast<unsigned char*>(base);
    if (b) {
        w.clip = reinterpret_cast<float*>(b + o_clip);
        w.dead = b + o_dead;
        w.st = reinterpret_cast<GpState*>(b + o_st);
        w.L = reinterpret_cast<double*>(b + o_L);
    }
    w.bytes = off;
    return w;
}

std::atomic<int> g_gptq_smem_set[kMaxDevices];

struct GemmIn {
    const void* x;
    int64_t M, K, ldx, N, ldy;
    float* y;
    int32_t* status;
    cudaStream_t stream;
    int qbits, wmode;                 // wmode 0: packed codes; 1 / 2: bf16 / fp32 weights + clip
    const uint8_t* packed;
    const uint16_t* scale;
    int64_t prb;
    bool tma_codes;
    const void* w;
    int64_t ldw;
    const float* clip;
    int export_scale;
};

// Decode-sized batches (M <= 16) of the dequant-on-load GEMM whose packed
// rows suit TMA: the register-level kernel of gq_gemm_decode.cuh over units
// of 256 weight rows x 512 of K, one block per SM; Y is zeroed first (the
// units add into it).
gq_status gemm_decode_launch(const void* d_x, int64_t M, int64_t K, int64_t ldx, const uint8_t* d_packed,
                             const uint16_t* d_scale_f16, int qbits, int64_t prb, int64_t N, float* d_y,
                             int64_t ldy, int32_t* d_status, cudaStream_t stream) {
    PFN_cuTensorMapEncodeTiled enc = encode_tiled();
    if (!enc) return GQ_ERR_UNSUPPORTED;
    DecParams P;
    std::memset(&P, 0, sizeof(P));
    const cuuint64_t gdim[2] = {(cuuint64_t)prb, (cuuint64_t)N};
    const cuuint64_t gstride[1] = {(cuuint64_t)prb};
    const cuuint32_t box[2] = {(cuuint32_t)(qbits == 6 ? dec_ss_bytes<6>() : dec_ss_bytes<8>()), 16u};
    const cuuint32_t estride[2] = {1, 1};
    if (enc(&P.tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(d_packed), gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return GQ_ERR_UNSUPPORTED;
    P.x = static_cast<const uint16_t*>(d_x);
    P.scale = d_scale_f16;
    P.y = d_y;
    P.status = d_status;
    P.ldx = ldx;
    P.ldy = ldy;
    P.M = M;
    P.N = N;
    P.K = K;
    P.kunits = (K + kDecKc - 1) / kDecKc;
    P.units = ((N + kDecRows - 1) / kDecRows) * P.kunits;
    const int64_t grid = std::min<int64_t>(sm_count(), P.units);
    if (cuda_status(cudaMemset2DAsync(d_y, (size_t)ldy * 4, 0, (size_t)N * 4, (size_t)M, stream)) != GQ_OK)
        return GQ_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQ_ERR_CUDA;
    const int qi = qbits == 6 ? 0 : 1;
    const int smem = qi ? dec_smem_bytes<8>() : dec_smem_bytes<6>();
    if (dev >= 0 && dev < kMaxDevices && g_dec_smem_set[qi][dev].load() < smem) {
        if (cuda_status(cudaFuncSetAttribute(qi ? gemm_decode_kernel<8> : gemm_decode_kernel<6>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != GQ_OK)
            return GQ_ERR_CUDA;
        g_dec_smem_set[qi][dev].store(smem);
    }
    if (qi == 0) gemm_decode_kernel<6><<<(unsigned)grid, kDecThreads, smem, stream>>>(P);
    else gemm_decode_kernel<8><<<(unsigned)grid, kDecThreads, smem, stream>>>(P);
    return launch_status();
}

// The launch shared by the dequant-on-load and the fake-quant-on-load GEMM
// (arguments already checked).
gq_status gemm_launch(const GemmIn& in) {
    const void* d_x = in.x;
    const int64_t M = in.M, K = in.K, ldx = in.ldx, N = in.N, ldy = in.ldy;
    float* d_y = in.y;
    int32_t* d_status = in.status;
    cudaStream_t stream = in.stream;
    const int qbits = in.qbits;
    const uint8_t* d_packed = in.packed;
    const uint16_t* d_scale_f16 = in.scale;
    const int64_t prb = in.prb;
    const bool tma_codes = in.tma_codes;
    PFN_cuTensorMapEncodeTiled enc = encode_tiled();
    if (!enc) return GQ_ERR_UNSUPPORTED;
    GemmParams P;
    std::memset(&P, 0, sizeof(P));
    // token tile: the batch itself up to 256 tokens (rounded up to 16 .. 256), else 256
    int nt = 16;
    while (nt < M && nt < 256) nt *= 2;
    P.nt = nt;
    P.ni = nt <= 64 ? 2 : 1;
    // K stages per code copy / W_hat chunk / MMA commit, and per X copy (at
    // most 32 KB); the weight modes copy one stage of weights at a time
    P.cs = in.wmode ? 1 : 4;
    P.xs = in.wmode ? 1 : nt <= 64 ? 4 : nt == 128 ? 2 : 1;
    P.wmode = in.wmode;
    P.idesc = gemm_idesc(kGemmBN, (uint32_t)nt);
    P.acc_cols = (uint32_t)std::max(32, nt);
    const cuuint32_t estride[3] = {1, 1, 1};
    // X: a 3-D view {64, M, K / 64} (one copy per chunk) when K % 64 == 0,
    // else the 2-D [M, K] view (one copy per stage)
    P.x3d = 0;
    if (K % kGemmBK == 0) {
        const cuuint64_t gdim3[3] = {(cuuint64_t)kGemmBK, (cuuint64_t)M, (cuuint64_t)(K / kGemmBK)};
        const cuuint64_t gstride3[2] = {(cuuint64_t)ldx * 2, (cuuint64_t)kGemmBK * 2};
        const cuuint32_t box3[3] = {(cuuint32_t)kGemmBK, (cuuint32_t)nt, (cuuint32_t)P.xs};
        if (enc(&P.tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(d_x), gdim3, gstride3, box3, estride,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            P.x3d = 1;
    }
    if (!P.x3d) {
        const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t gstride[1] = {(cuuint64_t)ldx * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kGemmBK, (cuuint32_t)nt};
        if (enc(&P.tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(d_x), gdim, gstride, box, estride,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return GQ_ERR_UNSUPPORTED;
    }
    // bytes of a row's 64-wide stage in a code slot (codes, or bf16 / fp32 weights)
    const int64_t cb = in.wmode == 1 ? 128 : in.wmode == 2 ? 256 : qbits == 6 ? 48 : 64;
    const int64_t crow = cb * P.cs;                   // ... of a row's chunk
    if (in.wmode == 1) {
        // bf16 weights [N, ldw]: box 64 x 128 (128-byte rows), 128-byte swizzle
        const cuuint64_t wdim[2] = {(cuuint64_t)K, (cuuint64_t)N};
        const cuuint64_t wstride[1] = {(cuuint64_t)in.ldw * 2};
        const cuuint32_t wbox[2] = {(cuuint32_t)kGemmBK, (cuuint32_t)kGemmBN};
        if (enc(&P.tmap_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(in.w), wdim, wstride, wbox, estride,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return GQ_ERR_UNSUPPORTED;
    } else if (in.wmode == 2) {
        // fp32 weights: a stage is two 32-wide halves (128-byte rows); one
        // 3-D copy {32, 128, 2} of the view {32, N, K / 32} when K % 32 == 0,
        // else two 2-D copies (the tail zero-filled)
        P.w3d = 0;
        if (K % 32 == 0) {
            const cuuint64_t wdim3[3] = {32, (cuuint64_t)N, (cuuint64_t)(K / 32)};
            const cuuint64_t wstride3[2] = {(cuuint64_t)in.ldw * 4, 128};
            const cuuint32_t wbox3[3] = {32, (cuuint32_t)kGemmBN, 2};
            if (enc(&P.tmap_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(in.w), wdim3, wstride3, wbox3,
                    estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
                P.w3d = 1;
        }
        if (!P.w3d) {
            const cuuint64_t wdim[2] = {(cuuint64_t)K, (cuuint64_t)N};
            const cuuint64_t wstride[1] = {(cuuint64_t)in.ldw * 4};
            const cuuint32_t wbox[2] = {32, (cuuint32_t)kGemmBN};
            if (enc(&P.tmap_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(in.w), wdim, wstride, wbox,
                    estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return GQ_ERR_UNSUPPORTED;
        }
    } else if (tma_codes) {
        const cuuint64_t wdim[2] = {(cuuint64_t)prb, (cuuint64_t)N};
        const cuuint64_t wstride[1] = {(cuuint64_t)prb};
        const cuuint32_t wbox[2] = {(cuuint32_t)crow, (cuuint32_t)kGemmBN};
        if (enc(&P.tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(d_packed), wdim, wstride, wbox,
                estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return GQ_ERR_UNSUPPORTED;
    }
    P.code_copy = (in.wmode == 0 && !tma_codes) ? 1 : 0;
    P.codes = d_packed;
    P.scale = d_scale_f16;
    P.clip = in.clip;
    P.export_scale = in.export_scale;
    P.y = d_y;
    P.status = d_status;
    P.M = M;
    P.N = N;
    P.K = K;
    P.ldy = ldy;
    P.prb = prb;
    P.qbits = qbits;
    P.kt_per_tile = (int32_t)((K + kGemmBK - 1) / kGemmBK);
    const int64_t tiles_n = (N + kGemmBN - 1) / kGemmBN, tiles_m = (M + nt - 1) / nt;
    P.tiles_m = (int32_t)tiles_m;
    P.tiles = tiles_n * tiles_m;
    const int64_t sms = sm_count();
    // few tiles: split the stage units evenly (partial sums added into a
    // zeroed Y); many: whole tiles round-robin
    P.streamk = P.tiles < 2 * sms ? 1 : 0;
    const int64_t units = P.streamk ? P.tiles * P.kt_per_tile : P.tiles;
    const int64_t grid = std::min<int64_t>(sms, units);
    // ring depths in chunks: X up to 64 KB (at least 2 slots), codes in what
    // is left, W_hat in the TMEM columns after the accumulators; the commit
    // ring is a multiple of the W_hat depth and at least the X depth (a
    // waiter on any of these barriers then never sees a phase two ahead)
    const int64_t x_bytes = (int64_t)nt * 128 * P.xs, c_bytes = kGemmBN * crow;
    // codes: 3 chunks (12 stages) for wide token tiles, else up to 6; X slots
    // in the rest (at most 8)
    const int64_t dc_want = in.wmode ? (in.wmode == 1 ? 6 : 4) : nt >= 128 ? 3 : 6;
    P.dc = (int32_t)std::min<int64_t>(dc_want, (kGemmRingBytes - 2 * x_bytes) / c_bytes);
    P.dx = (int32_t)std::min<int64_t>(in.wmode ? 12 : 8, (kGemmRingBytes - P.dc * c_bytes) / x_bytes);
    P.dw = (int32_t)std::min<int64_t>(kGemmMaxWS / P.cs, (512 - P.ni * (int64_t)P.acc_cols) / (32 * P.cs));
    P.dd = P.dw;                                        // the commit ring frees W_hat slots only
    if (P.dc < 2 || P.dw < 2 || P.dx < 2 || P.dd > kGemmMaxDone || P.dx > kGemmMaxX) return GQ_ERR_UNSUPPORTED;
    if (P.streamk &&
        cuda_status(cudaMemset2DAsync(d_y, (size_t)ldy * 4, 0, (size_t)N * 4, (size_t)M, stream)) != GQ_OK)
        return GQ_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQ_ERR_CUDA;
    const int wi = in.wmode ? 1 : 0;
    if (dev >= 0 && dev < kMaxDevices && g_gemm_smem_set[wi][dev].load() < kGemmSmemBytes) {
        if (cuda_status(cudaFuncSetAttribute(wi ? gemm_dequant_kernel<1> : gemm_dequant_kernel<0>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes)) != GQ_OK)
            return GQ_ERR_CUDA;
        g_gemm_smem_set[wi][dev].store(kGemmSmemBytes);
    }
    if (wi) gemm_dequant_kernel<1><<<(unsigned)grid, kGemmThreads, kGemmSmemBytes, stream>>>(P);
    else gemm_dequant_kernel<0><<<(unsigned)grid, kGemmThreads, kGemmSmemBytes, stream>>>(P);
    return launch_status();
}

}  // namespace

extern "C" {

size_t gq_gptq_workspace_size(int64_t rows, int64_t cols) {
    if (rows < 0 || cols < 0) return 0;
    return gptq_layout(nullptr, rows, cols).bytes;
}

gq_status gq_gptq_hessian(const void* d_x, int32_t dtype, int64_t n, int64_t cols, int64_t ldx, double* d_H,
                          int accumulate, cudaStream_t stream) {
    if (dtype != GQ_F32 && dtype != GQ_BF16) return GQ_ERR_INVALID_ARG;
    if (n < 0 || cols < 0 || ldx < cols || (accumulate != 0 && accumulate != 1)) return GQ_ERR_INVALID_ARG;
    if (cols == 0) return GQ_OK;
    if (!d_H || (n > 0 && !d_x)) return GQ_ERR_INVALID_ARG;
    if (cols > 65535 * (int64_t)kGpHTile || (n > 0 && n > INT64_MAX / 4 / ldx)) return GQ_ERR_UNSUPPORTED;
    if (!aligned(d_H, 8) || (n > 0 && !aligned(d_x, dtype == GQ_F32 ? 4 : 2))) return GQ_ERR_MISALIGNED;
    const unsigned tiles = (unsigned)((cols + kGpHTile - 1) / kGpHTile);
    gptq_hessian_kernel<<<dim3(tiles, tiles), kGpThreads, 0, stream>>>(d_x, dtype, n, cols, ldx, d_H, accumulate);
    return launch_status();
}

size_t gq_gptq_batch_workspace_size(const gq_tensor* t, int n) {
    if (!t || n <= 0) return 0;
    size_t total = 0;
    for (int i = 0; i < n; ++i) {
        if (t[i].rows < 0 || t[i].cols < 0) return 0;
        total += gptq_layout(nullptr, t[i].rows, t[i].cols).bytes;
    }
    return total;
}

gq_status gq_gptq_quantize_batch(const gq_tensor* t, int n, const double* const* d_H, double percdamp, void* d_ws,
                                 size_t ws_bytes, int32_t* d_status, cudaStream_t stream) {
    if (n < 0 || (n > 0 && (!t || !d_H))) return GQ_ERR_INVALID_ARG;
    if (!(percdamp >= 0.0 && percdamp < 1e6)) return GQ_ERR_INVALID_ARG;
    if (d_status && !aligned(d_status, 4)) return GQ_ERR_MISALIGNED;
    size_t need = 0;
    for (int i = 0; i < n; ++i) {
        const gq_tensor& T = t[i];
        gq_status st = check_tensor(T, Op::Export, true);
        if (st != GQ_OK) return st;
        if (T.qbits == 16 || T.gran != GQ_PER_ROW || T.col_scale) return GQ_ERR_UNSUPPORTED;
        if (T.rows == 0 || T.cols == 0) continue;
        if (!d_H[i]) return GQ_ERR_INVALID_ARG;
        if (!aligned(d_H[i], 8)) return GQ_ERR_MISALIGNED;
        if (T.cols > kGptqMaxCols) return GQ_ERR_UNSUPPORTED;
        need += gptq_layout(nullptr, T.rows, T.cols).bytes;
    }
    if (n == 0) return GQ_OK;
    if (need > 0) {
        if (!d_ws || ws_bytes < need) return GQ_ERR_WORKSPACE;
        if (!aligned(d_ws, 256)) return GQ_ERR_MISALIGNED;
    }
    if (d_status && cuda_status(cudaMemsetAsync(d_status, 0, sizeof(int32_t) * (size_t)n, stream)) != GQ_OK)
        return GQ_ERR_CUDA;
    // the non-empty weights, each with its part of the workspace
    std::vector<int> idx;
    std::vector<GptqWs> ws;
    size_t off = 0;
    for (int i = 0; i < n; ++i) {
        if (t[i].rows == 0 || t[i].cols == 0) continue;
        idx.push_back(i);
        ws.push_back(gptq_layout(static_cast<unsigned char*>(d_ws) + off, t[i].rows, t[i].cols));
        off += ws.back().bytes;
    }
    if (idx.empty()) return GQ_OK;
    const int nw = (int)idx.size();

    // 1. clip of every original row (the export's select), into the workspace
    std::vector<gq_tensor> sel(nw);
    for (int k = 0; k < nw; ++k) {
        sel[k] = t[idx[k]];
        sel[k].dq = nullptr;
        sel[k].codes = nullptr;
        sel[k].packed = nullptr;
        sel[k].scale_f16 = nullptr;
        sel[k].scale_f32 = nullptr;
        sel[k].clip = ws[k].clip;
    }
    if (nw == n) {
        // one batched select (status i is tensor i's)
        gq_status st = quantize_batch(sel.data(), nw, Op::Select, false, nullptr, 0, d_status, stream);
        if (st != GQ_OK) return st;
    } else {
        for (int k = 0; k < nw; ++k) {
            gq_status st = quantize_batch(&sel[k], 1, Op::Select, false, nullptr, 0,
                                          d_status ? d_status + idx[k] : nullptr, stream);
            if (st != GQ_OK) return st;
        }
    }
    for (int k = 0; k < nw; ++k) {
        const gq_tensor& T = t[idx[k]];
        if (T.clip && cuda_status(cudaMemcpyAsync(T.clip, ws[k].clip, (size_t)T.rows * 4, cudaMemcpyDeviceToDevice,
                                                  stream)) != GQ_OK)
            return GQ_ERR_CUDA;
    }
    // 2 - 4 in groups of kGpMaxMats weights
    const int64_t sms = sm_count();
    for (int g0 = 0; g0 < nw; g0 += kGpMaxMats) {
        const int gc = std::min(kGpMaxMats, nw - g0);
        GpMats M;
        std::memset(&M, 0, sizeof(M));
        M.count = gc;
        int64_t nmax = 0;
        for (int k = 0; k < gc; ++k) {
            const int i = idx[g0 + k];
            GpMat& G = M.m[k];
            G.H = d_H[i];
            G.L = ws[g0 + k].L;
            G.dead = ws[g0 + k].dead;
            G.st = ws[g0 + k].st;
            G.n = t[i].cols;
            nmax = std::max(nmax, G.n);
        }
        // 2. dead inputs, damping, reversal
        gptq_diag_kernel<<<(unsigned)gc, kGpThreads, 0, stream>>>(M, percdamp);
        const int64_t rev_blocks = std::min<int64_t>(
            std::max<int64_t>(1, sms * 8 / gc), (nmax * nmax + kGpThreads - 1) / kGpThreads);
        gptq_reverse_kernel<<<dim3((unsigned)rev_blocks, (unsigned)gc), kGpThreads, 0, stream>>>(M);
        if (launch_status() != GQ_OK) return GQ_ERR_CUDA;
        // 3. Cholesky of the reversed, damped Hessians, panel by panel
        for (int64_t k0 = 0; k0 < nmax; k0 += kGpBlock) {
            const int64_t below = std::max<int64_t>(0, nmax - k0 - kGpBlock);
            const unsigned pblocks = (unsigned)std::max<int64_t>(1, (below + 63) / 64);
            gptq_chol_panel<<<dim3(pblocks, 1, (unsigned)gc), kGpThreads, 0, stream>>>(M, k0);
            if (below > 0) {
                const unsigned ut = (unsigned)((below + 63) / 64);
                gptq_chol_update<<<dim3(ut, ut, (unsigned)gc), kGpThreads, 0, stream>>>(M, k0);
            }
            if (launch_status() != GQ_OK) return GQ_ERR_CUDA;
        }
        // 4. the recurrence over the rows of every weight of the group: one
        // launch per shared-memory class (blocks per SM that the residuals of
        // a weight's columns allow), so that narrow weights are not given the
        // shared memory, and the occupancy, of the widest
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return GQ_ERR_CUDA;
        auto per_sm = [](int64_t cols) { return (int)std::min<int64_t>(8, 232448 / (int64_t)gptq_rows_smem(cols)); };
        std::vector<int> classes;
        for (int k = 0; k < gc; ++k) {
            const int c = per_sm(t[idx[g0 + k]].cols);
            if (std::find(classes.begin(), classes.end(), c) == classes.end()) classes.push_back(c);
        }
        std::sort(classes.begin(), classes.end());            // the widest weights first
        for (int cls : classes) {
            GptqParams P;
            std::memset(&P, 0, sizeof(P));
            int64_t blocks = 0, ncls = 0;
            int nd = 0;
            for (int k = 0; k < gc; ++k) {
                const int i = idx[g0 + k];
                const gq_tensor& T = t[i];
                if (per_sm(T.cols) != cls) continue;
                GptqRowDesc& R = P.d[nd++];
                R.w = T.w;
                R.L = ws[g0 + k].L;
                R.dead = ws[g0 + k].dead;
                R.st = ws[g0 + k].st;
                R.clip = ws[g0 + k].clip;
                R.scale_f16 = T.scale_f16;
                R.codes = T.codes;
                R.packed = T.packed;
                R.dq = T.dq;
                R.status = d_status ? d_status + i : nullptr;
                R.rows = T.rows;
                R.n = T.cols;
                R.ld = T.ld;
                R.prb = packed_row_bytes(T.cols, T.qbits);
                R.start = blocks;
                R.dtype = T.dtype;
                R.qbits = T.qbits;
                blocks += (T.rows + kGpRows - 1) / kGpRows;
                ncls = std::max(ncls, T.cols);
            }
            P.ndesc = nd;
            P.blocks = blocks;
            if (P.blocks > INT32_MAX) return GQ_ERR_UNSUPPORTED;
            const size_t smem = gptq_rows_smem(ncls);
            if (dev >= 0 && dev < kMaxDevices && g_gptq_smem_set[dev].load() < (int)smem) {
                if (cuda_status(cudaFuncSetAttribute(gptq_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)smem)) != GQ_OK)
                    return GQ_ERR_CUDA;
                g_gptq_smem_set[dev].store((int)smem);
            }
            gptq_rows_kernel<<<(unsigned)P.blocks, kGpThreads, smem, stream>>>(P);
            if (launch_status() != GQ_OK) return GQ_ERR_CUDA;
        }
    }
    return GQ_OK;
}

gq_status gq_gptq_quantize(const gq_tensor* t, const double* d_H, double percdamp, void* d_ws, size_t ws_bytes,
                           int32_t* d_status, cudaStream_t stream) {
    if (!t) return GQ_ERR_INVALID_ARG;
    return gq_gptq_quantize_batch(t, 1, &d_H, percdamp, d_ws, ws_bytes, d_status, stream);
}

gq_status gq_row_clip_select(const gq_tensor* t, int n, void* d_ws, size_t ws_bytes,
                             int32_t* d_status, cudaStream_t stream) {
    return quantize_batch(t, n, Op::Select, false, d_ws, ws_bytes, d_status, stream);
}

gq_status gq_fakequant_fwd(const gq_tensor* t, int n, gq_scale_mode mode, void* d_ws,
                           size_t ws_bytes, int32_t* d_status, cudaStream_t stream) {
    if (mode != GQ_SCALE_F32 && mode != GQ_SCALE_F16) return GQ_ERR_INVALID_ARG;
    return quantize_batch(t, n, Op::FakeQuant, mode == GQ_SCALE_F16, d_ws, ws_bytes, d_status,
                          stream);
}

gq_status gq_fakequant_average(const gq_tensor* t, const gq_avg* avg, int n, gq_scale_mode mode,
                               void* d_ws, size_t ws_bytes, int32_t* d_status, cudaStream_t stream) {
    if (mode != GQ_SCALE_F32 && mode != GQ_SCALE_F16) return GQ_ERR_INVALID_ARG;
    return quantize_batch(t, n, Op::Average, mode == GQ_SCALE_F16, d_ws, ws_bytes, d_status, stream, avg);
}

gq_status gq_export_pack(const gq_tensor* t, int n, void* d_ws, size_t ws_bytes,
                         int32_t* d_status, cudaStream_t stream) {
    return quantize_batch(t, n, Op::Export, true, d_ws, ws_bytes, d_status, stream);
}

gq_status gq_export_pack_noalloc(const gq_tensor* t, int n, int32_t* d_status,
                                 cudaStream_t stream) {
    if (n < 0 || (n > 0 && !t)) return GQ_ERR_INVALID_ARG;
    const size_t need = n > 0 ? workspace_size(t, n, false) : 0;   // no candidate buffers here
    if (need > kNoAllocBytes) return GQ_ERR_WORKSPACE;
    void* ws = nullptr;
    if (need > 0) {
        gq_status st = noalloc_scratch(&ws);
        if (st != GQ_OK) return st;
    }
    return quantize_batch(t, n, Op::Export, true, ws, kNoAllocBytes, d_status, stream, nullptr, false);
}

gq_status gq_test_arm_wait_expiry(int64_t tile, uint64_t wait_ns) {
    if (tile < 0 || wait_ns < 1000000ull || wait_ns > kWaitLimitNs) return GQ_ERR_INVALID_ARG;
    g_test_poison_tile = tile;
    g_test_wait_ns = wait_ns;
    return GQ_OK;
}

gq_status gq_ste_bwd(const void* d_g_out, void* d_g_w, gq_dtype dtype, int64_t numel,
                     int accumulate, cudaStream_t stream) {
    if (dtype != GQ_F32 && dtype != GQ_BF16) return GQ_ERR_INVALID_ARG;
    if (numel < 0 || (accumulate != 0 && accumulate != 1)) return GQ_ERR_INVALID_ARG;
    if (numel == 0) return GQ_OK;
    if (!d_g_out || !d_g_w) return GQ_ERR_INVALID_ARG;
    const size_t esz = dtype == GQ_F32 ? 4 : 2;
    if (!aligned(d_g_out, esz) || !aligned(d_g_w, esz)) return GQ_ERR_MISALIGNED;
    if ((uint64_t)numel > (uint64_t)INT64_MAX / 16) return GQ_ERR_INVALID_ARG;
    const int vec = aligned(d_g_out, 16) && aligned(d_g_w, 16);
    const int64_t per = dtype == GQ_F32 ? 4 : 8;
    const int64_t units = vec ? (numel + per - 1) / per : numel;
    const int64_t blocks = std::min<int64_t>((int64_t)sm_count() * 8,
                                             std::max<int64_t>(1, (units + kBlockThreads - 1) / kBlockThreads));
    ste_kernel<<<(unsigned)blocks, kBlockThreads, 0, stream>>>(d_g_out, d_g_w, dtype, numel,
                                                                accumulate, vec);
    return launch_status();
}

gq_status gq_dequant(const uint8_t* d_packed, const uint16_t* d_scale_f16, int qbits,
                     gq_gran gran, int64_t rows, int64_t cols, void* d_out,
                     gq_dtype out_dtype, cudaStream_t stream) {
    if (qbits != 6 && qbits != 8) return GQ_ERR_INVALID_ARG;
    if (gran != GQ_PER_ROW && gran != GQ_PER_TENSOR) return GQ_ERR_INVALID_ARG;
    if (out_dtype != GQ_F32 && out_dtype != GQ_BF16) return GQ_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0) return GQ_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return GQ_OK;
    if (!d_packed || !d_scale_f16 || !d_out) return GQ_ERR_INVALID_ARG;
    if (rows > INT64_MAX / 16 / cols) return GQ_ERR_INVALID_ARG;
    const size_t esz = out_dtype == GQ_F32 ? 4 : 2;
    if (!aligned(d_scale_f16, 2) || !aligned(d_out, esz)) return GQ_ERR_MISALIGNED;
    const int64_t prb = packed_row_bytes(cols, qbits);
    const size_t vin = out_dtype == GQ_F32 ? 16 : 8;
    const int vec_out = aligned(d_out, vin) && ((cols * (int64_t)esz) % (int64_t)vin) == 0;
    const int words = aligned(d_packed, 4) && (qbits == 6 ? (cols % 16) == 0 : (cols % 4) == 0);
    // one warp per row segment of 32 * kDqUnroll quads (the kernel's work items)
    const int64_t segs = ((cols + 3) / 4 + 32 * kDqUnroll - 1) / (32 * kDqUnroll);
    const int64_t blocks = std::min<int64_t>((int64_t)sm_count() * 8,
                                             (rows * segs + kBlockWarps - 1) / kBlockWarps);
    dequant_kernel<<<(unsigned)blocks, kBlockThreads, 0, stream>>>(
        d_packed, d_scale_f16, qbits, gran == GQ_PER_TENSOR, rows, cols, prb, d_out, out_dtype,
        vec_out, words);
    return launch_status();
}

gq_status gq_gemm_dequant(const void* d_x, int64_t M, int64_t K, int64_t ldx, const uint8_t* d_packed,
                          const uint16_t* d_scale_f16, int qbits, int64_t N, float* d_y, int64_t ldy,
                          int32_t* d_status, cudaStream_t stream) {
    if (M < 0 || N < 0 || K < 0 || (qbits != 6 && qbits != 8)) return GQ_ERR_INVALID_ARG;
    if (ldx < K || ldy < N) return GQ_ERR_INVALID_ARG;
    if (M > INT32_MAX || K > INT32_MAX || N > INT32_MAX) return GQ_ERR_UNSUPPORTED;
    const int64_t prb = packed_row_bytes(K, qbits);
    const bool tma_codes = prb % 16 == 0;
    if (!tma_codes && prb % 4 != 0) return GQ_ERR_UNSUPPORTED;   // int6 needs K % 16 == 0, int8 K % 4 == 0
    if (d_status && !aligned(d_status, 4)) return GQ_ERR_MISALIGNED;
    if (d_status && cuda_status(cudaMemsetAsync(d_status, 0, sizeof(int32_t), stream)) != GQ_OK) return GQ_ERR_CUDA;
    if (M == 0 || N == 0) return GQ_OK;
    if (!d_x || !d_packed || !d_scale_f16 || !d_y) return GQ_ERR_INVALID_ARG;
    if (!aligned(d_x, 16) || (ldx % 8) != 0 || !aligned(d_packed, tma_codes ? 16 : 4) ||
        !aligned(d_scale_f16, 2) || !aligned(d_y, 4))
        return GQ_ERR_MISALIGNED;
    if (K == 0)
        return cuda_status(cudaMemset2DAsync(d_y, (size_t)ldy * 4, 0, (size_t)N * 4, (size_t)M, stream));
    if (M <= kDecMaxM && tma_codes)
        return gemm_decode_launch(d_x, M, K, ldx, d_packed, d_scale_f16, qbits, prb, N, d_y, ldy, d_status, stream);
    GemmIn in{};
    in.x = d_x; in.M = M; in.K = K; in.ldx = ldx; in.N = N; in.y = d_y; in.ldy = ldy; in.status = d_status;
    in.stream = stream; in.qbits = qbits; in.wmode = 0; in.packed = d_packed; in.scale = d_scale_f16;
    in.prb = prb; in.tma_codes = tma_codes;
    return gemm_launch(in);
}

gq_status gq_gemm_fakequant(const void* d_x, int64_t M, int64_t K, int64_t ldx, const void* d_w, int32_t w_dtype,
                            int64_t ldw, const float* d_clip, int qbits, gq_scale_mode mode, int64_t N, float* d_y,
                            int64_t ldy, int32_t* d_status, cudaStream_t stream) {
    if (M < 0 || N < 0 || K < 0 || (qbits != 6 && qbits != 8)) return GQ_ERR_INVALID_ARG;
    if (w_dtype != GQ_F32 && w_dtype != GQ_BF16) return GQ_ERR_INVALID_ARG;
    if (mode != GQ_SCALE_F32 && mode != GQ_SCALE_F16) return GQ_ERR_INVALID_ARG;
    if (ldx < K || ldw < K || ldy < N) return GQ_ERR_INVALID_ARG;
    if (M > INT32_MAX || K > INT32_MAX || N > INT32_MAX) return GQ_ERR_UNSUPPORTED;
    if (d_status && !aligned(d_status, 4)) return GQ_ERR_MISALIGNED;
    if (d_status && cuda_status(cudaMemsetAsync(d_status, 0, sizeof(int32_t), stream)) != GQ_OK) return GQ_ERR_CUDA;
    if (M == 0 || N == 0) return GQ_OK;
    if (!d_x || !d_w || !d_clip || !d_y) return GQ_ERR_INVALID_ARG;
    const int64_t esz = w_dtype == GQ_F32 ? 4 : 2;
    if (!aligned(d_x, 16) || (ldx % 8) != 0 || !aligned(d_w, 16) || ((ldw * esz) % 16) != 0 || !aligned(d_clip, 4) ||
        !aligned(d_y, 4))
        return GQ_ERR_MISALIGNED;
    if (K == 0)
        return cuda_status(cudaMemset2DAsync(d_y, (size_t)ldy * 4, 0, (size_t)N * 4, (size_t)M, stream));
    GemmIn in{};
    in.x = d_x; in.M = M; in.K = K; in.ldx = ldx; in.N = N; in.y = d_y; in.ldy = ldy; in.status = d_status;
    in.stream = stream; in.qbits = qbits; in.wmode = w_dtype == GQ_BF16 ? 1 : 2; in.w = d_w; in.ldw = ldw;
    in.clip = d_clip; in.export_scale = mode == GQ_SCALE_F16 ? 1 : 0;
    return gemm_launch(in);
}

size_t gq_workspace_size(const gq_tensor* t, int n) {
    if (!t || n <= 0) return 0;
    return workspace_size(t, n);
}

int64_t gq_packed_row_bytes(int64_t cols, int qbits) { return packed_row_bytes(cols, qbits); }

int64_t gq_k_from_p(int64_t n, double p) {
    if (n < 1 || !(p > 0.0 && p <= 1.0)) return -1;
    return k_from_p(n, p);
}

int gq_plan_kind(const char* name, const int64_t* shape, int ndim, int is_float,
                 const char* patterns, int64_t small_numel) {
    if (!name || ndim < 0 || (ndim > 0 && !shape) || small_numel < 0) return -1;
    int64_t numel = 1;
    for (int i = 0; i < ndim; ++i) {
        if (shape[i] < 0) return -1;
        numel *= shape[i];
    }
    if (!is_float) return GQ_KIND_RAW;
    if (numel < small_numel) return GQ_KIND_FP16;
    const char* pats = patterns ? patterns : "tok_emb.weight,lm_head.weight";
    const char* p = pats;
    while (*p) {
        const char* comma = std::strchr(p, ',');
        size_t len = comma ? (size_t)(comma - p) : std::strlen(p);
        // trim spaces
        const char* b = p;
        const char* e = p + len;
        while (b < e && *b == ' ') ++b;
        while (e > b && e[-1] == ' ') --e;
        if (e > b) {
            std::string pat(b, (size_t)(e - b));
            if (std::strstr(name, pat.c_str())) return GQ_KIND_INT8;
        }
        if (!comma) break;
        p = comma + 1;
    }
    return GQ_KIND_INT6;
}

int gq_last_cuda_error(void) { return g_last_cuda_error; }

const char* gq_last_cuda_error_string(void) {
    return g_last_cuda_error ? cudaGetErrorString((cudaError_t)g_last_cuda_error) : "no error";
}

const char* gq_status_string(gq_status s) {
    switch (s) {
        case GQ_OK: return "ok";
        case GQ_ERR_INVALID_ARG: return "invalid argument";
        case GQ_ERR_UNSUPPORTED: return "unsupported";
        case GQ_ERR_MISALIGNED: return "misaligned pointer";
        case GQ_ERR_WORKSPACE: return "workspace missing or too small";
        case GQ_ERR_RANGE: return "binary16 scale overflow";
        case GQ_ERR_NONFINITE: return "non-finite input";
        case GQ_ERR_CUDA: return "CUDA error";
        case GQ_ERR_TIMEOUT: return "timeout";
    }
    return "unknown status";
}

}  // extern "C"
