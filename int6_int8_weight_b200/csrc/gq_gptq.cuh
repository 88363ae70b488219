// gq_gptq.cuh -- GPTQ-lite on the GPU: column-by-column quantization of a
// weight [rows, n] with error feedback through the Hessian H [n, n] of its
// inputs, on the per-row grid of the export (binary16 row scales from the
// percentile clip of the original row).  Source: "Record: Unified Attention +
// FA3 + Legal TTT" (PR #1202), section Quantization ("GPTQ-lite, bits 6");
// the method is the published GPTQ algorithm (Frantar et al. 2022,
// Algorithm 1).  Everything runs in binary64 on the CUDA cores: the kernels
// are bound by double-precision FMA throughput, and binary64 keeps every
// code decision on the same side of its rounding boundary as a binary64
// reference.
//
// Formulation.  GPTQ quantizes column j after feeding forward the errors of
// the columns before it.  With U the upper Cholesky factor of H^-1 and E the
// scaled errors, its updates satisfy W = Q + E U, so E = (W - Q) U^-1.
// U^-1 =: V is upper triangular with V V^T = H (a Cholesky factorization of
// H in reversed index order), and the value that column j is rounded from is
//     w~_j = w_j + sum_{i < j} (w_i - q_i s) V[i, j] / V[j, j],
// a left-looking recurrence over the ORIGINAL weights and the residuals
// r_i = w_i - q_i s.  No inverse is formed: V comes from one Cholesky
// factorization of the damped H with its rows and columns reversed,
// Hr = P H P = L L^T, V[i, j] = L[n-1-i, n-1-j].
//
// Kernels (one launch each unless noted):
//   gptq_hessian_kernel  H (+)= 2 X^T X, 64 x 64 tiles of the lower
//                        triangle, mirrored;
//   gptq_diag_kernel     dead inputs (zero diagonal) and the damping
//                        lambda = percdamp * mean(diag);
//   gptq_reverse_kernel  Hr = P (H + lambda I) P into the workspace, with
//                        dead diagonals set to 1 first;
//   gptq_chol_panel / gptq_chol_update  right-looking blocked Cholesky of
//                        Hr in place (2 launches per 64-wide panel);
//   gptq_rows_kernel     the recurrence, 4 rows per block, columns in
//                        batches of 64: a dot-product pass over the earlier
//                        columns' residuals, then the batch's columns in
//                        order (one warp per row, one shuffle per column);
//                        writes codes, packed rows, w_hat and scales.
#pragma once

#include "gq_device.cuh"

namespace gq {

constexpr int kGpBlock = 64;         // columns per batch of the recurrence / Cholesky panel width
constexpr int kGpRows = 4;           // weight rows per block of the recurrence
constexpr int kGpThreads = 256;
constexpr int kGpHTile = 64;         // Hessian tile
constexpr int kGpHChunk = 32;        // input rows per Hessian step

// ------------------------------------------------------------- Hessian --

__device__ __forceinline__ double gp_load(const void* x, int dtype, int64_t idx) {
    if (dtype == kF32) return (double)reinterpret_cast<const float*>(x)[idx];
    return (double)bf16_bits_to_float(reinterpret_cast<const uint16_t*>(x)[idx]);
}

// H[i, j] (+)= 2 sum_t x[t, i] x[t, j] for the 64 x 64 tile (blockIdx.y,
// blockIdx.x) of the lower triangle; the tile is mirrored into the upper
// triangle.  Thread (ty, tx) owns the 4 x 4 entries 4 ty + a, 4 tx + b.
__global__ void __launch_bounds__(kGpThreads) gptq_hessian_kernel(const void* __restrict__ x, int dtype,
                                                                  int64_t n, int64_t cols, int64_t ldx,
                                                                  double* __restrict__ H, int accumulate) {
    const int ti = blockIdx.y, tj = blockIdx.x;
    if (tj > ti) return;
    __shared__ double xi[kGpHChunk][kGpHTile + 1];
    __shared__ double xj[kGpHChunk][kGpHTile + 1];
    const int t = threadIdx.x, ty = t / 16, tx = t % 16;
    const int64_t i0 = (int64_t)ti * kGpHTile, j0 = (int64_t)tj * kGpHTile;
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
    for (int64_t r0 = 0; r0 < n; r0 += kGpHChunk) {
        for (int e = t; e < kGpHChunk * kGpHTile; e += kGpThreads) {
            const int rr = e / kGpHTile, cc = e % kGpHTile;
            const int64_t r = r0 + rr;
            xi[rr][cc] = (r < n && i0 + cc < cols) ? gp_load(x, dtype, r * ldx + i0 + cc) : 0.0;
            xj[rr][cc] = (r < n && j0 + cc < cols) ? gp_load(x, dtype, r * ldx + j0 + cc) : 0.0;
        }
        __syncthreads();
#pragma unroll 4
        for (int rr = 0; rr < kGpHChunk; ++rr) {
            double a4[4], b4[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) a4[a] = xi[rr][4 * ty + a];
#pragma unroll
            for (int b = 0; b < 4; ++b) b4[b] = xj[rr][4 * tx + b];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = __fma_rn(a4[a], b4[b], acc[a][b]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int64_t i = i0 + 4 * ty + a, j = j0 + 4 * tx + b;
            if (i < cols && j < cols && j <= i) {
                const double v = 2.0 * acc[a][b];
                H[i * cols + j] = accumulate ? H[i * cols + j] + v : v;
                if (i != j) H[j * cols + i] = H[i * cols + j];
            }
        }
}

// ------------------------------------------------- damping and reversal --

struct GpState {
    double lambda;       // damping added to the diagonal
    int32_t dead_count;
    int32_t bad;         // non-finite or non-positive pivot met
};

// The per-weight matrices of a batch: the kernels below take their matrix
// from a grid index, so that the independent chains of several weights run
// in the same launches.
struct GpMat {
    const double* H;     // [n, n] Hessian (input)
    double* L;           // [n, n] reversed, damped Hessian, then its lower factor
    uint8_t* dead;       // [n]
    GpState* st;
    int64_t n;
};
constexpr int kGpMaxMats = 64;
struct GpMats {
    int32_t count;
    int32_t pad;
    GpMat m[kGpMaxMats];
};

// One block per matrix: dead inputs (H[j, j] == 0 -> flagged, treated as 1)
// and lambda = percdamp * mean(diag H) over the fixed diagonal.
__global__ void __launch_bounds__(kGpThreads) gptq_diag_kernel(const __grid_constant__ GpMats M, double percdamp) {
    const GpMat& G = M.m[blockIdx.x];
    const double* __restrict__ H = G.H;
    const int64_t n = G.n;
    uint8_t* __restrict__ dead = G.dead;
    GpState* st = G.st;
    __shared__ double part[kGpThreads];
    __shared__ int cnt[kGpThreads];
    double sum = 0.0;
    int c = 0;
    for (int64_t j = threadIdx.x; j < n; j += kGpThreads) {
        const double d = H[j * n + j];
        const bool z = d == 0.0;
        dead[j] = z ? 1 : 0;
        sum += z ? 1.0 : d;
        c += z ? 1 : 0;
    }
    part[threadIdx.x] = sum;
    cnt[threadIdx.x] = c;
    __syncthreads();
    for (int w = kGpThreads / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) {
            part[threadIdx.x] += part[threadIdx.x + w];
            cnt[threadIdx.x] += cnt[threadIdx.x + w];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        st->lambda = percdamp * (part[0] / (double)n);
        st->dead_count = cnt[0];
        st->bad = 0;
    }
}

// Hr[a, b] = Hd[n-1-a, n-1-b] for b <= a, Hd = H with dead diagonals set to 1
// and lambda added to the diagonal (a dead input also drops out of the
// off-diagonal coupling: its weights are zeroed, so its row of H is unused).
// (matrix blockIdx.y of the batch; the x blocks stride over its entries)
__global__ void __launch_bounds__(kGpThreads) gptq_reverse_kernel(const __grid_constant__ GpMats M) {
    const GpMat& G = M.m[blockIdx.y];
    const double* __restrict__ H = G.H;
    const int64_t n = G.n;
    const uint8_t* __restrict__ dead = G.dead;
    double* __restrict__ Hr = G.L;
    const double lam = G.st->lambda;
    const int64_t total = n * n;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t a = e / n, b = e % n;
        if (b > a) continue;
        const int64_t i = n - 1 - a, j = n - 1 - b;
        double v = H[i * n + j];
        if (a == b) v = (dead[i] ? 1.0 : v) + lam;
        Hr[a * n + b] = v;
    }
}

// ------------------------------------------------------------ Cholesky --

// Panel k0 (width nb = min(64, n - k0)) of the lower Cholesky factor, in
// place: every block factors the diagonal block in shared memory (the
// trailing updates of earlier panels are already applied), block 0 writes it
// back, and each block solves 64 rows below it: L[i, k0 + c] =
// (A[i, k0 + c] - sum_{d < c} L[i, k0 + d] L[k0 + c, k0 + d]) / L[k0 + c, k0 + c].
// (matrix blockIdx.z of the batch; a matrix whose order is at most k0 has no
// panel here, and x blocks past its own row count do nothing)
__global__ void __launch_bounds__(kGpThreads) gptq_chol_panel(const __grid_constant__ GpMats M, int64_t k0) {
    const GpMat& G = M.m[blockIdx.z];
    const int64_t n = G.n;
    if (k0 >= n) return;
    if ((int64_t)blockIdx.x * 64 >= max((int64_t)1, n - k0 - kGpBlock)) return;
    double* __restrict__ A = G.L;
    GpState* st = G.st;
    __shared__ double D[kGpBlock][kGpBlock + 1];
    const int nb = (int)min((int64_t)kGpBlock, n - k0);
    const int t = threadIdx.x;
    for (int e = t; e < nb * nb; e += kGpThreads) {
        const int r = e / nb, c = e % nb;
        D[r][c] = c <= r ? A[(k0 + r) * n + k0 + c] : 0.0;
    }
    __syncthreads();
    for (int j = 0; j < nb; ++j) {
        if (t == 0) {
            const double d = D[j][j];
            if (!(d > 0.0)) st->bad = 1;           // not positive definite (or NaN)
            D[j][j] = sqrt(d);
        }
        __syncthreads();
        const double piv = D[j][j];
        for (int r = j + 1 + t; r < nb; r += kGpThreads) D[r][j] = D[r][j] / piv;
        __syncthreads();
        // rank-1 update of the block's trailing lower triangle
        const int m = nb - j - 1;
        for (int e = t; e < m * m; e += kGpThreads) {
            const int r = j + 1 + e / m, c = j + 1 + e % m;
            if (c <= r) D[r][c] = __fma_rn(-D[r][j], D[c][j], D[r][c]);
        }
        __syncthreads();
    }
    if (blockIdx.x == 0)
        for (int e = t; e < nb * nb; e += kGpThreads) {
            const int r = e / nb, c = e % nb;
            if (c <= r) A[(k0 + r) * n + k0 + c] = D[r][c];
        }
    // rows below the diagonal block: one row per thread group of 4 (each
    // thread takes one row; 64 rows per block)
    const int64_t i = k0 + nb + (int64_t)blockIdx.x * 64 + t;
    if (t < 64 && i < n) {
        double row[kGpBlock];
#pragma unroll 8
        for (int c = 0; c < nb; ++c) row[c] = A[i * n + k0 + c];
        for (int c = 0; c < nb; ++c) {
            double v = row[c];
            for (int d = 0; d < c; ++d) v = __fma_rn(-row[d], D[c][d], v);
            row[c] = v / D[c][c];
        }
#pragma unroll 8
        for (int c = 0; c < nb; ++c) A[i * n + k0 + c] = row[c];
    }
}

// Trailing update after panel k0: A[i, j] -= sum_c L[i, k0 + c] L[j, k0 + c]
// for k0 + nb <= j <= i, on 64 x 64 tiles of the lower triangle; the panel
// columns are staged 32 at a time.
// (matrix blockIdx.z of the batch; tiles past its own trailing block do nothing)
__global__ void __launch_bounds__(kGpThreads) gptq_chol_update(const __grid_constant__ GpMats M, int64_t k0) {
    const GpMat& G = M.m[blockIdx.z];
    const int64_t n = G.n;
    const int ti = blockIdx.y, tj = blockIdx.x;
    if (tj > ti || k0 + kGpBlock >= n) return;
    double* __restrict__ A = G.L;
    const int nb = kGpBlock;
    const int64_t base = k0 + nb;
    if (base + (int64_t)ti * 64 >= n) return;
    const int64_t i0 = base + (int64_t)ti * 64, j0 = base + (int64_t)tj * 64;
    constexpr int kCh = 32;
    __shared__ double Pi[64][kCh + 1];
    __shared__ double Pj[64][kCh + 1];
    const int t = threadIdx.x, ty = t / 16, tx = t % 16;
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
    for (int c0 = 0; c0 < nb; c0 += kCh) {
        for (int e = t; e < 64 * kCh; e += kGpThreads) {
            const int r = e / kCh, c = e % kCh;
            const bool in = c0 + c < nb;
            Pi[r][c] = (i0 + r < n && in) ? A[(i0 + r) * n + k0 + c0 + c] : 0.0;
            Pj[r][c] = (j0 + r < n && in) ? A[(j0 + r) * n + k0 + c0 + c] : 0.0;
        }
        __syncthreads();
        for (int c = 0; c < kCh; ++c) {
            double a4[4], b4[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) a4[a] = Pi[4 * ty + a][c];
#pragma unroll
            for (int b = 0; b < 4; ++b) b4[b] = Pj[4 * tx + b][c];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = __fma_rn(a4[a], b4[b], acc[a][b]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int64_t i = i0 + 4 * ty + a, j = j0 + 4 * tx + b;
            if (i < n && j <= i) A[i * n + j] -= acc[a][b];
        }
}

// ---------------------------------------------------------- recurrence --

struct GptqRowDesc {
    const void* w;
    const double* L;         // lower Cholesky factor of the reversed, damped Hessian [n, n]
    const uint8_t* dead;     // [n]
    const GpState* st;
    const float* clip;       // [rows] percentile clip of the original rows
    uint16_t* scale_f16;     // [rows] out
    int8_t* codes;           // [rows, n] out, nullable
    uint8_t* packed;         // [rows, prb] out
    void* dq;                // [rows, n] out (w's dtype), nullable
    int32_t* status;         // nullable
    int64_t rows, n, ld, prb;
    int64_t start;           // first block of this descriptor in the launch
    int32_t dtype, qbits;
};

constexpr int kGpMaxDesc = kGpMaxMats;

struct GptqParams {
    int32_t ndesc;
    int64_t blocks;
    GptqRowDesc d[kGpMaxDesc];
};

// Shared memory of gptq_rows_kernel: residuals of the block's rows over all
// columns [kGpRows][n], the batch's scaled factor block [64][65], the
// partial sums [kGpRows][64] and the batch's codes [kGpRows][64].
__host__ __device__ inline size_t gptq_rows_smem(int64_t n) {
    return (size_t)kGpRows * (size_t)n * 8 + (size_t)kGpBlock * (kGpBlock + 1) * 8 + (size_t)kGpRows * kGpBlock * 8 +
           (size_t)kGpRows * kGpBlock * 4;
}

__global__ void __launch_bounds__(kGpThreads) gptq_rows_kernel(const __grid_constant__ GptqParams P) {
    extern __shared__ __align__(16) unsigned char gp_smem[];
    int di = 0;
    while (di + 1 < P.ndesc && (int64_t)blockIdx.x >= P.d[di + 1].start) ++di;
    const GptqRowDesc& D = P.d[di];
    const int64_t n = D.n;
    const int64_t r0 = ((int64_t)blockIdx.x - D.start) * kGpRows;
    const int nr = (int)min((int64_t)kGpRows, D.rows - r0);
    double* res = reinterpret_cast<double*>(gp_smem);                     // [kGpRows][n]
    double* Mb = res + (size_t)kGpRows * n;                                // [64][65]
    double* part = Mb + kGpBlock * (kGpBlock + 1);                         // [kGpRows][64]
    int* qs = reinterpret_cast<int*>(part + kGpRows * kGpBlock);           // [kGpRows][64]
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int qmax = D.qbits == 6 ? 31 : 127;
    const double* L = D.L;

    // row scales: the export's, from the clip of the original row
    __shared__ double c_row[kGpRows], s_row[kGpRows];
    if (t < kGpRows) {
        c_row[t] = 0.0;
        s_row[t] = 0.0;
        if (t < nr) {
            uint16_t h;
            bool range;
            const Scale S = make_scale(__float_as_uint(D.clip[r0 + t]), qmax, true, &h, &range);
            c_row[t] = (double)S.c;
            s_row[t] = (double)S.s;
            D.scale_f16[r0 + t] = h;
            if (range && D.status) atomicOr(reinterpret_cast<unsigned int*>(D.status), 0x2u);
        }
    }
    if (t == 0 && D.st->bad && D.status) atomicOr(reinterpret_cast<unsigned int*>(D.status), 0x1u);
    __syncthreads();

    for (int64_t j0 = 0; j0 < n; j0 += kGpBlock) {
        const int nb = (int)min((int64_t)kGpBlock, n - j0);
        // (a) the earlier columns' contribution: thread (r, jj) sums
        // res[r, i] * L[n-1-i, n-1-j] over i < j0, divided by V[j, j] below
        {
            const int r = t / kGpBlock, jj = t % kGpBlock;
            double acc = 0.0;
            if (r < nr && jj < nb) {
                const int64_t colL = n - 1 - (j0 + jj);
                const double* rr = res + (size_t)r * n;
                for (int64_t i = 0; i < j0; ++i) acc = __fma_rn(rr[i], L[(n - 1 - i) * n + colL], acc);
            }
            part[r * kGpBlock + jj] = acc;
        }
        // the batch's own factor block, scaled by its column's diagonal:
        // Mb[ii][jj] = V[j0+ii, j0+jj] / V[j0+jj, j0+jj] for ii < jj
        for (int e = t; e < kGpBlock * kGpBlock; e += kGpThreads) {
            const int ii = e / kGpBlock, jj = e % kGpBlock;
            double v = 0.0;
            if (ii < jj && jj < nb) {
                const int64_t a = n - 1 - (j0 + ii), b = n - 1 - (j0 + jj);
                v = L[a * n + b] / L[b * n + b];
            }
            Mb[ii * (kGpBlock + 1) + jj] = v;
        }
        __syncthreads();
        // (b) the batch's columns in order: warp r owns row r, lane owns
        // columns lane and lane + 32 of the batch
        if (warp < nr) {
            const int r = warp;
            const int64_t grow = r0 + r;
            double acc2[2], wv[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int jj = lane + 32 * h;
                const int64_t j = j0 + jj;
                double base = 0.0;
                if (jj < nb) {
                    const double vjj = L[(n - 1 - j) * n + (n - 1 - j)];
                    base = part[r * kGpBlock + jj] / vjj;
                    wv[h] = D.dead[j] ? 0.0 : gp_load(D.w, D.dtype, grow * D.ld + j);
                } else {
                    wv[h] = 0.0;
                }
                acc2[h] = base;
            }
            for (int jj = 0; jj < nb; ++jj) {
                const int h = jj >> 5, owner = jj & 31;
                double resid = 0.0;
                int q = 0;
                if (lane == owner) {
                    const double wj = h ? wv[1] : wv[0];
                    const double wt = wj + (h ? acc2[1] : acc2[0]);
                    const double s = s_row[r], c = c_row[r];
                    double qd = 0.0;
                    if (s != 0.0) {
                        const double vc = fmin(fmax(wt, -c), c);
                        qd = fmin(fmax(rint(vc / s), (double)-qmax), (double)qmax);
                    }
                    q = (int)qd;
                    resid = wj - qd * s;
                    qs[r * kGpBlock + jj] = q;
                    res[(size_t)r * n + j0 + jj] = resid;
                }
                resid = __shfl_sync(0xFFFFFFFFu, resid, owner);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int c2 = lane + 32 * hh;
                    if (c2 > jj && c2 < nb) acc2[hh] = __fma_rn(resid, Mb[jj * (kGpBlock + 1) + c2], acc2[hh]);
                }
            }
        }
        __syncthreads();
        // (c) outputs of the batch: codes, w_hat, packed bytes
        for (int e = t; e < kGpRows * kGpBlock; e += kGpThreads) {
            const int r = e / kGpBlock, jj = e % kGpBlock;
            if (r >= nr || jj >= nb) continue;
            const int64_t grow = r0 + r, j = j0 + jj;
            const int q = qs[r * kGpBlock + jj];
            if (D.codes) D.codes[grow * n + j] = (int8_t)q;
            if (D.dq) {
                const float v = q == 0 ? 0.0f : __fmul_rn((float)q, (float)s_row[r]);
                if (D.dtype == kF32) reinterpret_cast<float*>(D.dq)[grow * n + j] = v;
                else reinterpret_cast<uint16_t*>(D.dq)[grow * n + j] = float_to_bf16_bits(v);
            }
            if (D.qbits == 8) D.packed[grow * D.prb + j] = (uint8_t)(int8_t)q;
        }
        if (D.qbits == 6) {
            // 4 codes -> 3 bytes; batches are 64 wide, so groups never straddle
            for (int e = t; e < kGpRows * (kGpBlock / 4); e += kGpThreads) {
                const int r = e / (kGpBlock / 4), g = e % (kGpBlock / 4);
                if (r >= nr || 4 * g >= nb) continue;
                uint32_t v = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int jj = 4 * g + k;
                    const uint32_t u = jj < nb ? ((uint32_t)qs[r * kGpBlock + jj] & 0x3Fu) : 0u;
                    v |= u << (6 * k);
                }
                uint8_t* dst = D.packed + (r0 + r) * D.prb + 3 * ((j0 + 4 * g) / 4);
                dst[0] = (uint8_t)(v & 0xFF);
                dst[1] = (uint8_t)((v >> 8) & 0xFF);
                dst[2] = (uint8_t)((v >> 16) & 0xFF);
            }
        }
        __syncthreads();
    }
}

}  // namespace gq
