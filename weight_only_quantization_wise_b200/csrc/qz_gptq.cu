// qz_gptq.cu -- GPTQ layer-wise quantization (GPTQ explainer, azimuth.plus/paper/gptq).
//
// The page's algorithm for one linear layer: from calibration data X (one
// column per sample) form H = 2 X X^T, add a small damping term lambda I,
// take the Cholesky decomposition of H^-1 once, then quantize the weight
// columns in one fixed order for every row; after each column, every weight
// not yet quantized is moved to compensate that column's rounding error
// (OBQ's update, read from the Cholesky factor), and the updates are batched
// lazily in blocks of B = 128 columns: inside a block they are applied at
// once, the rest of the matrix gets one large matrix update per block.  The
// output is the packed format of qz_quantize_pack (codes, bf16 scales,
// zeros), so the decode GEMV and the prefill GEMM consume it unchanged.
//
// Arithmetic.  Everything but the quantizer runs in fp64, like the CPU
// reference this library is checked against; a group's scale and zero and
// every code come from the fp64 weights rounded to fp32, with the fp32
// operations of qz_quantize_pack (IEEE division, round half to even), so
// codes agree with the reference unless a compensated weight lies within
// about 1e-16 of a rounding boundary.
//
// Steps and kernels (U is the upper Cholesky factor of the damped H^-1):
//   1. hessian_kernel: R = 2 X X^T + lambda I with rows and columns in
//      reverse order (R[a][b] = H[K-1-a][K-1-b]); lambda = damp * mean of
//      the diagonal (1 when that mean is 0), added by damp_kernel.
//   2. Blocked Cholesky R = L L^T (L lower, 64 x 64 tiles): chol_diag_kernel
//      factors a diagonal tile, chol_panel_kernel solves the tiles below it,
//      chol_update_kernel updates the trailing lower triangle.
//      Reversing both indices turns L into an upper V with H = V V^T, so
//      H^-1 = V^-T V^-1 and V^-1 is upper: it is U.
//   3. Blocked inverse Li = L^-1: trinv_diag_kernel inverts the diagonal
//      tiles; then, right-looking, for each block row m trinv_finalize_kernel
//      completes row m (Li[m,j] = -Li[m,m] sum_{k<m} L[m,k] Li[k,j]) and
//      trinv_update_kernel adds row m's contribution to every later row, so
//      each launch has many independent tiles; reverse_kernel writes
//      U[j][k] = Li[K-1-j][K-1-k].
//   4. Per block of 128 columns: gptq_block_kernel (one warp per weight row,
//      the row's 128 block columns in registers, U's block triangle in
//      shared memory) quantizes the columns in order, applies the
//      in-block updates and records the scaled errors E; then
//      lazy_update_kernel applies W[:, end:] -= E U[block, end:].
#include <cuda_runtime.h>

#include <math.h>

#include "qz_internal.cuh"

namespace qz {
namespace {

constexpr int kT = 64;              // tile edge of the factorization kernels
constexpr int kTileThreads = 256;   // 16 x 16 threads, 4 x 4 outputs each
constexpr int kGptqBlock = 128;     // the page's lazy-batch width B
constexpr int kRowsPerCta = 32;     // warps (weight rows) per column-loop CTA

// ---------------------------------------------------------------------------
// fp64 tile product helper: acc (4 x 4 per thread of a 16 x 16 layout over a
// 64 x 64 tile) += As (64 x kT) * Bs (kT x 64), both in shared memory.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tile_fma(double (&acc)[4][4], const double (*As)[kT + 1],
                                         const double (*Bs)[kT + 1], int ty, int tx, int kd) {
    for (int k = 0; k < kd; ++k) {
        double a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[ty + 16 * i][k];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
}

// Two padded 64 x 64 fp64 tiles (66.5 KB) live in dynamic shared memory.
using Tile = double[kT][kT + 1];
constexpr size_t kTwoTiles = 2 * sizeof(Tile);
#define QZ_TWO_TILES(As, Bs)                                     \
    extern __shared__ double qz_tiles_[];                        \
    Tile &As = *reinterpret_cast<Tile *>(qz_tiles_);             \
    Tile &Bs = *reinterpret_cast<Tile *>(qz_tiles_ + kT * (kT + 1))

__device__ __forceinline__ double bf16_to_f64(uint16_t h) {
    return (double)__uint_as_float((uint32_t)h << 16);
}

// 1. R[a][b] = 2 sum_t x[t][K-1-a] x[t][K-1-b] for the tiles on or below the
// diagonal (the factorization reads only the lower triangle).
__global__ void __launch_bounds__(kTileThreads)
hessian_kernel(const uint16_t *__restrict__ x, int64_t n_samples, int K, double *__restrict__ R) {
    const int bi = blockIdx.y, bj = blockIdx.x;
    if (bj > bi) return;
    QZ_TWO_TILES(As, Bs);               // As [row a][sample], Bs [sample][col b]
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    double acc[4][4] = {};
    for (int64_t t0 = 0; t0 < n_samples; t0 += kT) {
        const int kd = (int)(n_samples - t0 < kT ? n_samples - t0 : kT);
        for (int e = tid; e < kT * kT; e += kTileThreads) {
            const int r = e / kT, c = e % kT;          // r: feature in tile, c: sample
            const int ga = bi * kT + r, gb = bj * kT + r;
            const bool ok = c < kd;
            As[r][c] = (ok && ga < K) ? bf16_to_f64(x[(t0 + c) * K + (K - 1 - ga)]) : 0.0;
            Bs[c][r] = (ok && gb < K) ? bf16_to_f64(x[(t0 + c) * K + (K - 1 - gb)]) : 0.0;
        }
        __syncthreads();
        tile_fma(acc, As, Bs, ty, tx, kd);
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int a = bi * kT + ty + 16 * i, b = bj * kT + tx + 16 * j;
            if (a < K && b < K) R[(int64_t)a * K + b] = 2.0 * acc[i][j];
        }
}

// lambda = damp * mean(diag), or 1 when the mean is 0; added to the diagonal.
__global__ void damp_kernel(double *R, int K, double damp) {
    __shared__ double part[256];
    double s = 0.0;
    for (int a = threadIdx.x; a < K; a += blockDim.x) s += R[(int64_t)a * K + a];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    const double mean = part[0] / (double)K;
    const double lambda = mean > 0.0 ? damp * mean : 1.0;
    for (int a = threadIdx.x; a < K; a += blockDim.x) R[(int64_t)a * K + a] += lambda;
}

// 2a. Factor the diagonal tile p in place (unblocked Cholesky in shared
// memory); the strict upper part of the tile is zeroed.  Thread t owns row
// t / 4 and, within it, the columns c = t % 4 (mod 4), so each step touches
// only the trailing triangle.
__global__ void __launch_bounds__(kTileThreads) chol_diag_kernel(double *R, int K, int p) {
    __shared__ double A[kT][kT + 1];
    const int base = p * kT, n = min(kT, K - base);
    for (int e = threadIdx.x; e < kT * kT; e += kTileThreads) {
        const int r = e / kT, c = e % kT;
        A[r][c] = (r < n && c < n) ? R[(int64_t)(base + r) * K + base + c] : 0.0;
    }
    __syncthreads();
    const int i = threadIdx.x >> 2, cls = threadIdx.x & 3;
    for (int j = 0; j < n; ++j) {
        if (threadIdx.x == 0) A[j][j] = sqrt(A[j][j]);
        __syncthreads();
        if (cls == 0 && i > j && i < n) A[i][j] /= A[j][j];
        __syncthreads();
        // trailing update: A[i][c] -= A[i][j] A[c][j], j < c <= i
        if (i > j && i < n) {
            const double aij = A[i][j];
            int c = j + 1 + ((cls - (j + 1)) & 3);
            for (; c <= i; c += 4) A[i][c] -= aij * A[c][j];
        }
        __syncthreads();
    }
    for (int e = threadIdx.x; e < kT * kT; e += kTileThreads) {
        const int r = e / kT, c = e % kT;
        if (r < n && c < n) R[(int64_t)(base + r) * K + base + c] = c <= r ? A[r][c] : 0.0;
    }
}

// 2b. Tiles below the diagonal in panel p: A[i,p] <- A[i,p] L[p,p]^-T.  Row r
// of a tile solves x L^T = b column by column: x_c = b_c / L[c][c], then
// b_k -= x_c L[k][c] for k > c (the same operations, in the same order, as
// the forward substitution x_c = (b_c - sum_{k<c} x_k L[c][k]) / L[c][c]).
// Thread t owns row t % 64 and the columns k = t / 64 (mod 4).
__global__ void __launch_bounds__(kTileThreads) chol_panel_kernel(double *R, int K, int p) {
    QZ_TWO_TILES(Lp, B);
    const int base = p * kT, n = min(kT, K - base);
    const int rb = (p + 1 + blockIdx.x) * kT, rows = min(kT, K - rb);
    for (int e = threadIdx.x; e < kT * kT; e += kTileThreads) {
        const int r = e / kT, c = e % kT;
        Lp[r][c] = (r < n && c < n) ? R[(int64_t)(base + r) * K + base + c] : 0.0;
        B[r][c] = (r < rows && c < n) ? R[(int64_t)(rb + r) * K + base + c] : 0.0;
    }
    __syncthreads();
    const int r = threadIdx.x & (kT - 1), cls = threadIdx.x / kT;
    for (int c = 0; c < n; ++c) {
        if ((c & 3) == cls && r < rows) B[r][c] /= Lp[c][c];
        __syncthreads();
        if (r < rows) {
            const double x = B[r][c];
            for (int k = c + 1 + ((cls - (c + 1)) & 3); k < n; k += 4) B[r][k] -= x * Lp[k][c];
        }
        __syncthreads();
    }
    for (int e = threadIdx.x; e < kT * kT; e += kTileThreads) {
        const int rr = e / kT, c = e % kT;
        if (rr < rows && c < n) R[(int64_t)(rb + rr) * K + base + c] = B[rr][c];
    }
}

// 2c. Trailing update of the tiles (i, j), p < j <= i:
// A[i,j] -= A[i,p] A[j,p]^T.  Block (x, y) of the grid maps to i = p+1+y,
// j = p+1+x; tiles above the diagonal return at once.
__global__ void __launch_bounds__(kTileThreads) chol_update_kernel(double *R, int K, int p) {
    const int i = p + 1 + blockIdx.y, j = p + 1 + blockIdx.x;
    if (j > i) return;
    QZ_TWO_TILES(As, Bs);
    const int base = p * kT, n = min(kT, K - base);
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    for (int e = tid; e < kT * kT; e += kTileThreads) {
        const int r = e / kT, c = e % kT;
        const int gi = i * kT + r, gj = j * kT + r;
        As[r][c] = (gi < K && c < n) ? R[(int64_t)gi * K + base + c] : 0.0;
        Bs[c][r] = (gj < K && c < n) ? R[(int64_t)gj * K + base + c] : 0.0;
    }
    __syncthreads();
    double acc[4][4] = {};
    tile_fma(acc, As, Bs, ty, tx, n);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int gi = i * kT + ty + 16 * a, gj = j * kT + tx + 16 * b;
            if (gi < K && gj < K && gj <= gi) R[(int64_t)gi * K + gj] -= acc[a][b];
        }
}

// 3a. Invert each diagonal tile of L: Li[p,p] = L[p,p]^-1 (column by column
// forward substitution, one thread per column).
__global__ void __launch_bounds__(kTileThreads)
trinv_diag_kernel(const double *__restrict__ L, double *__restrict__ Li, int K) {
    QZ_TWO_TILES(A, X);
    const int p = blockIdx.x, base = p * kT, n = min(kT, K - base);
    for (int e = threadIdx.x; e < kT * kT; e += kTileThreads) {
        const int r = e / kT, c = e % kT;
        A[r][c] = (r < n && c < n) ? L[(int64_t)(base + r) * K + base + c] : 0.0;
    }
    __syncthreads();
    if ((int)threadIdx.x < n) {
        const int c = threadIdx.x;
        for (int i = 0; i < n; ++i) {
            if (i < c) {
                X[i][c] = 0.0;
                continue;
            }
            double v = (i == c) ? 1.0 : 0.0;
            for (int k = c; k < i; ++k) v -= A[i][k] * X[k][c];
            X[i][c] = v / A[i][i];
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kT * kT; e += kTileThreads) {
        const int r = e / kT, c = e % kT;
        if (r < n && c < n) Li[(int64_t)(base + r) * K + base + c] = X[r][c];
    }
}

// 3b. Off-diagonal tiles, right-looking: with S[i,j] = sum_{m<i} L[i,m] Li[m,j]
// accumulated in place of Li[i,j] (zero to start), step m first finalizes
// block row m, Li[m,j] = -Li[m,m] S[m,j] for j < m (trinv_finalize_kernel),
// then adds L[i,m] Li[m,j] to S[i,j] for every i > m, j <= m
// (trinv_update_kernel): all tiles of a step are independent.
__global__ void __launch_bounds__(kTileThreads)
trinv_finalize_kernel(double *__restrict__ Li, int K, int m) {
    const int j = blockIdx.x;
    QZ_TWO_TILES(As, Bs);
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    for (int e = tid; e < kT * kT; e += kTileThreads) {
        const int r = e / kT, c = e % kT;
        const int gr = m * kT + r, gc = m * kT + c, gj = j * kT + c;
        As[r][c] = (gr < K && gc < K) ? Li[(int64_t)gr * K + gc] : 0.0;
        Bs[r][c] = (gr < K && gj < K) ? Li[(int64_t)gr * K + gj] : 0.0;
    }
    __syncthreads();
    double out[4][4] = {};
    tile_fma(out, As, Bs, ty, tx, kT);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int gi = m * kT + ty + 16 * a, gj = j * kT + tx + 16 * b;
            if (gi < K && gj < K) Li[(int64_t)gi * K + gj] = -out[a][b];
        }
}

__global__ void __launch_bounds__(kTileThreads)
trinv_update_kernel(const double *__restrict__ L, double *__restrict__ Li, int K, int m) {
    const int j = blockIdx.x, i = m + 1 + blockIdx.y;
    QZ_TWO_TILES(As, Bs);
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    for (int e = tid; e < kT * kT; e += kTileThreads) {
        const int r = e / kT, c = e % kT;
        const int gi = i * kT + r, gm = m * kT + c, gmr = m * kT + r, gj = j * kT + c;
        As[r][c] = (gi < K && gm < K) ? L[(int64_t)gi * K + gm] : 0.0;
        Bs[r][c] = (gmr < K && gj < K) ? Li[(int64_t)gmr * K + gj] : 0.0;
    }
    __syncthreads();
    double acc[4][4] = {};
    tile_fma(acc, As, Bs, ty, tx, kT);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int gi = i * kT + ty + 16 * a, gj = j * kT + tx + 16 * b;
            if (gi < K && gj < K) Li[(int64_t)gi * K + gj] += acc[a][b];
        }
}

// U[j][k] = Li[K-1-j][K-1-k].
__global__ void reverse_kernel(const double *__restrict__ Li, double *__restrict__ U, int K) {
    const int64_t total = (int64_t)K * K;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x)
        U[e] = Li[total - 1 - e];
}

// bf16 weights -> fp64 working copy.
__global__ void widen_kernel(const uint16_t *__restrict__ w, double *__restrict__ W, int64_t total) {
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x)
        W[e] = bf16_to_f64(w[e]);
}

// ---------------------------------------------------------------------------
// Quantizer (the fp32 arithmetic of qz_quantize_pack, on fp32 values).
// ---------------------------------------------------------------------------
struct Format {
    int bits, symmetric, qmin, qmax;
};

__device__ __forceinline__ uint32_t f32_bf16_up(float s) {
    const uint32_t b = __float_as_uint(s);
    uint32_t kept = b & 0xFFFF0000u;
    if (b & 0x0000FFFFu) kept += 0x00010000u;
    return kept >> 16;
}

// Scale (bf16 bits) and zero-point of a group from its range: vmin <= 0 <= vmax
// (asymmetric) or amax = max |x| (symmetric).
__device__ __forceinline__ void scale_zero(const Format &f, float vmin, float vmax, float amax,
                                           uint32_t &sb, int &z) {
    float S = f.symmetric ? __fdiv_rn(amax, (float)f.qmax)
                          : __fdiv_rn(__fsub_rn(vmax, vmin), (float)(f.qmax - f.qmin));
    if (S == 0.0f) S = 1.0f;
    sb = f32_bf16_up(S);
    const float Sf = __uint_as_float(sb << 16);
    z = f.symmetric ? 0 : f.qmin - (int)rintf(__fdiv_rn(vmin, Sf));
}

__device__ __forceinline__ int code_of(const Format &f, float x, uint32_t sb, int z) {
    const float Sf = __uint_as_float(sb << 16);
    const float u = __fadd_rn(__fdiv_rn(x, Sf), (float)z);
    int c = (int)rintf(u);
    c = c < f.qmin ? f.qmin : c;
    return c > f.qmax ? f.qmax : c;
}

__device__ __forceinline__ double warp_min(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmin(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}
__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// 4a. One block of columns [c0, c0 + nb) for kRowsPerCta weight rows, one
// warp per row: lane l holds columns c0 + l + 32 i (i = 0..3) in registers.
// U's block triangle (U[c0 + a][c0 + b], a <= b) sits in shared memory.
struct BlockArgs {
    double *W;                 // N x K working weights (fp64)
    double *E;                 // N x 128 scaled errors of the block
    const double *U;           // K x K
    uint8_t *codes;
    uint16_t *scales;
    uint8_t *zeros;
    int N, K, g, c0, nb;
    Format f;
};

__global__ void __launch_bounds__(32 * kRowsPerCta) gptq_block_kernel(const BlockArgs p) {
    extern __shared__ double Ut[];            // [nb][nb], row-major (upper part used)
    const int nb = p.nb;
    for (int e = threadIdx.x; e < nb * nb; e += blockDim.x) {
        const int a = e / nb, b = e % nb;
        Ut[e] = b >= a ? p.U[(int64_t)(p.c0 + a) * p.K + p.c0 + b] : 0.0;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * kRowsPerCta + warp;
    if (row >= p.N) return;
    double *Wr = p.W + (int64_t)row * p.K;
    double w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int c = lane + 32 * i;
        w[i] = c < nb ? Wr[p.c0 + c] : 0.0;
    }
    const int gpr = p.K / p.g;
    uint32_t sb = 0;
    int z = 0;
    if (p.c0 % p.g != 0) {
        // the block starts inside a group whose first column an earlier
        // block (launch) quantized: its stored scale and zero apply
        const int64_t e = (int64_t)row * gpr + p.c0 / p.g;
        sb = p.scales[e];
        z = p.f.symmetric ? 0
                          : (p.f.bits == 4 ? (int)p.zeros[e] : (int)(int8_t)p.zeros[e]);
    }
    uint32_t pending = 0;                     // int4: the low nibble of the byte being built
    for (int j = 0; j < nb; ++j) {
        const int col = p.c0 + j;
        if (col % p.g == 0) {
            // a group starts: its range from the current weights (inside the
            // block from registers; a group longer than the block reads the
            // rest of the row, which is current at a block start)
            float vmin = 0.0f, vmax = 0.0f, amax = 0.0f;
            const int gend = col + p.g;
            for (int c = col + lane; c < gend; c += 32) {
                const int lc = c - p.c0;
                double v;
                if (lc < nb) {
                    const int i = lc >> 5;
                    v = i == 0 ? w[0] : i == 1 ? w[1] : i == 2 ? w[2] : w[3];
                } else {
                    v = Wr[c];
                }
                const float vf = __double2float_rn(v);
                vmin = fminf(vmin, vf);
                vmax = fmaxf(vmax, vf);
                amax = fmaxf(amax, fabsf(vf));
            }
            vmin = (float)warp_min((double)vmin);
            vmax = (float)warp_max((double)vmax);
            amax = (float)warp_max((double)amax);
            scale_zero(p.f, vmin, vmax, amax, sb, z);
            if (lane == 0) {
                p.scales[(int64_t)row * gpr + col / p.g] = (uint16_t)sb;
                if (!p.f.symmetric) p.zeros[(int64_t)row * gpr + col / p.g] = (uint8_t)(int8_t)z;
            }
        }
        const int owner = j & 31, slot = j >> 5;
        const double mine = slot == 0 ? w[0] : slot == 1 ? w[1] : slot == 2 ? w[2] : w[3];
        const double wj = __shfl_sync(0xFFFFFFFFu, mine, owner);
        const int q = code_of(p.f, __double2float_rn(wj), sb, z);
        const double w_hat = (double)__uint_as_float(sb << 16) * (double)(q - z);
        const double e = (wj - w_hat) / Ut[j * nb + j];
        if (lane == 0) {
            p.E[(int64_t)row * kGptqBlock + j] = e;
            if (p.f.bits == 8) {
                p.codes[(int64_t)row * p.K + col] = (uint8_t)(int8_t)q;
            } else if ((col & 1) == 0) {
                pending = (uint32_t)q & 0xFu;
            } else {
                p.codes[(int64_t)row * (p.K / 2) + col / 2] =
                    (uint8_t)(pending | (((uint32_t)q & 0xFu) << 4));
            }
        }
        // w_k -= e * U[j][k], rounded twice (product, then difference) as the
        // reference does
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int c = lane + 32 * i;
            if (c > j && c < nb) w[i] = __dsub_rn(w[i], __dmul_rn(e, Ut[j * nb + c]));
        }
    }
}

// 4b. W[:, c0 + 128 :] -= E (N x nb) * U[c0 .. c0 + nb, c0 + 128 :]: 64 x 64
// output tiles, fp64.
__global__ void __launch_bounds__(kTileThreads)
lazy_update_kernel(double *__restrict__ W, const double *__restrict__ E,
                   const double *__restrict__ U, int N, int K, int c0, int nb) {
    const int r0 = blockIdx.y * kT, k0 = c0 + nb + blockIdx.x * kT;
    QZ_TWO_TILES(As, Bs);
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    double acc[4][4] = {};
    for (int j0 = 0; j0 < nb; j0 += kT) {
        const int kd = min(kT, nb - j0);
        for (int e = tid; e < kT * kT; e += kTileThreads) {
            const int r = e / kT, c = e % kT;
            As[r][c] = (r0 + r < N && c < kd) ? E[(int64_t)(r0 + r) * kGptqBlock + j0 + c] : 0.0;
            Bs[r][c] = (r < kd && k0 + c < K) ? U[(int64_t)(c0 + j0 + r) * K + k0 + c] : 0.0;
        }
        __syncthreads();
        tile_fma(acc, As, Bs, ty, tx, kd);
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int r = r0 + ty + 16 * a, k = k0 + tx + 16 * b;
            if (r < N && k < K) W[(int64_t)r * K + k] -= acc[a][b];
        }
}

struct Workspace {
    double *R, *Li, *W, *E;
};

Workspace carve(void *ws, int64_t N, int64_t K) {
    auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
    char *p = static_cast<char *>(ws);
    Workspace w;
    w.R = reinterpret_cast<double *>(p);
    p += up((size_t)K * K * sizeof(double));
    w.Li = reinterpret_cast<double *>(p);
    p += up((size_t)K * K * sizeof(double));
    w.W = reinterpret_cast<double *>(p);
    p += up((size_t)N * K * sizeof(double));
    w.E = reinterpret_cast<double *>(p);
    return w;
}

unsigned grid_for(int64_t total) {
    const int64_t b = (total + 255) / 256;
    return (unsigned)(b < (int64_t)device_sm_count() * 16 ? (b < 1 ? 1 : b)
                                                          : (int64_t)device_sm_count() * 16);
}

}  // namespace

size_t gptq_workspace_bytes(int64_t N, int64_t K) {
    auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
    return 2 * up((size_t)K * K * sizeof(double)) + up((size_t)N * K * sizeof(double)) +
           up((size_t)N * kGptqBlock * sizeof(double));
}

qz_status launch_gptq(const void *w, const void *x, int64_t N, int64_t K, int64_t n_samples,
                      int bits, int symmetric, int64_t group_size, double damp, void *codes,
                      void *scales, void *zeros, void *workspace, cudaStream_t st) {
    const Workspace ws = carve(workspace, N, K);
    const int Ki = (int)K, P = (int)((K + kT - 1) / kT);
    const size_t block_smem = (size_t)kGptqBlock * kGptqBlock * sizeof(double);
    static DeviceOnce attr_once;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return QZ_ERR_CUDA;
    }
    if (attr_once.run(dev, [block_smem] {
            const cudaFuncAttribute a = cudaFuncAttributeMaxDynamicSharedMemorySize;
            cudaError_t e = cudaFuncSetAttribute(hessian_kernel, a, (int)kTwoTiles);
            if (e == cudaSuccess) e = cudaFuncSetAttribute(chol_panel_kernel, a, (int)kTwoTiles);
            if (e == cudaSuccess) e = cudaFuncSetAttribute(chol_update_kernel, a, (int)kTwoTiles);
            if (e == cudaSuccess) e = cudaFuncSetAttribute(trinv_diag_kernel, a, (int)kTwoTiles);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(trinv_finalize_kernel, a, (int)kTwoTiles);
            if (e == cudaSuccess) e = cudaFuncSetAttribute(trinv_update_kernel, a, (int)kTwoTiles);
            if (e == cudaSuccess) e = cudaFuncSetAttribute(lazy_update_kernel, a, (int)kTwoTiles);
            if (e == cudaSuccess) e = cudaFuncSetAttribute(gptq_block_kernel, a, (int)block_smem);
            return e;
        }) != cudaSuccess)
        return QZ_ERR_CUDA;
    // 1. damped Hessian, reversed order
    hessian_kernel<<<dim3(P, P), kTileThreads, kTwoTiles, st>>>(
        static_cast<const uint16_t *>(x), n_samples, Ki, ws.R);
    damp_kernel<<<1, 256, 0, st>>>(ws.R, Ki, damp);
    // 2. Cholesky R = L L^T
    for (int p = 0; p < P; ++p) {
        chol_diag_kernel<<<1, kTileThreads, 0, st>>>(ws.R, Ki, p);
        if (p + 1 < P) {
            chol_panel_kernel<<<P - p - 1, kTileThreads, kTwoTiles, st>>>(ws.R, Ki, p);
            chol_update_kernel<<<dim3(P - p - 1, P - p - 1), kTileThreads, kTwoTiles, st>>>(
                ws.R, Ki, p);
        }
    }
    // 3. Li = L^-1, then U (reversed)
    if (cudaMemsetAsync(ws.Li, 0, (size_t)K * K * sizeof(double), st) != cudaSuccess)
        return QZ_ERR_CUDA;
    trinv_diag_kernel<<<P, kTileThreads, kTwoTiles, st>>>(ws.R, ws.Li, Ki);
    for (int m = 0; m < P; ++m) {
        if (m > 0) trinv_finalize_kernel<<<m, kTileThreads, kTwoTiles, st>>>(ws.Li, Ki, m);
        if (m + 1 < P)
            trinv_update_kernel<<<dim3(m + 1, P - m - 1), kTileThreads, kTwoTiles, st>>>(
                ws.R, ws.Li, Ki, m);
    }
    double *U = ws.R;   // the factor is no longer needed
    reverse_kernel<<<grid_for(K * K), 256, 0, st>>>(ws.Li, U, Ki);
    // 4. column loop
    widen_kernel<<<grid_for(N * K), 256, 0, st>>>(static_cast<const uint16_t *>(w), ws.W, N * K);
    BlockArgs a;
    a.W = ws.W;
    a.E = ws.E;
    a.U = U;
    a.codes = static_cast<uint8_t *>(codes);
    a.scales = static_cast<uint16_t *>(scales);
    a.zeros = static_cast<uint8_t *>(zeros);
    a.N = (int)N;
    a.K = Ki;
    a.g = (int)group_size;
    a.f.bits = bits;
    a.f.symmetric = symmetric;
    code_range(bits, symmetric, &a.f.qmin, &a.f.qmax);
    const unsigned row_ctas = (unsigned)((N + kRowsPerCta - 1) / kRowsPerCta);
    for (int c0 = 0; c0 < Ki; c0 += kGptqBlock) {
        a.c0 = c0;
        a.nb = Ki - c0 < kGptqBlock ? Ki - c0 : kGptqBlock;
        gptq_block_kernel<<<row_ctas, 32 * kRowsPerCta, (size_t)a.nb * a.nb * sizeof(double),
                            st>>>(a);
        const int rest = Ki - c0 - a.nb;
        if (rest > 0)
            lazy_update_kernel<<<dim3((rest + kT - 1) / kT, (unsigned)((N + kT - 1) / kT)),
                                 kTileThreads, kTwoTiles, st>>>(ws.W, ws.E, U, (int)N, Ki, c0,
                                                                a.nb);
    }
    return launch_status();
}

}  // namespace qz
