// rq_gptq.cu -- GPTQ on the symmetric group-64 grid.
//
// The "Hakureirm/rwkv7-sglang-w4gptq-1.5b" model card (opening summary)
// quantizes with GPTQ calibration into the same symmetric group-64 format as
// its calibration-free RTN variant; "rwkv-quant: uma matriz em bf16 elimina
// 39% das perdas na quantização do RWKV-7 2.9B" ("Vazamento de calibração e
// medições honestas") runs GPTQ on the preset's grid without changing the
// format, the kernels or the file size.  The method is the published GPTQ
// (Frantar et al., arXiv:2210.17323): the columns of W are quantized in order
// and each column's rounding error is spread over the columns not yet
// quantized, weighted through U, the upper Cholesky factor of the damped
// inverse Hessian of the layer input (H = 2 X^T X / T, H^-1 = U^T U).
//
// Three steps, each its own entry point:
//   hessian   H = (2/T) X^T X in fp64 (tiled, every element summed over t in
//             order);
//   factor    dead inputs (H[j][j] == 0: H[j][j] = 1, flagged), damping
//             H += damp * mean(diag H) * I, then U from the identity
//             U = P L^-1 P, where P reverses the index order and L is the lower
//             Cholesky factor of P H P (so H^-1 = P L^-T L^-1 P = U^T U with U
//             upper); fp64 throughout, U rounded to fp32 at the end.  The
//             Cholesky is right-looking, one launch per column; the triangular
//             inverse runs one warp per column of L^-1;
//   quantize  the column loop in fp32, in blocks of 128 columns: an in-block
//             kernel (one warp per row: lane l holds columns 4l..4l+3 of the
//             block, the block's 128 x 128 corner of U in shared memory) finds
//             each group's scale from the current weights when the loop
//             reaches the group's first column (fp32 amax / qmax, fp16 round
//             to nearest even: the RTN scale), takes the RTN code of each
//             column against it, and spreads its error e_j = (w_j - c_j s16) /
//             U[j][j] over the block's later columns with fmaf(-e_j, U[j][k],
//             w_k); a trailing kernel then applies the block's 128 errors to
//             every later column, per element in ascending j with the same
//             fmaf.  Every element therefore sees exactly the operations of a
//             sequential column loop, in the same order: the codes and scales
//             are bit-exact with a scalar fp32 implementation of that loop.
//             A group whose scale is unusable (non-finite weight: 0x7E00,
//             status NONFINITE; fp16 overflow: 0x7C00, status RANGE) gets
//             codes 0 and spreads no error.
#include <cuda_fp16.h>

#include "rq_internal.h"

namespace rq {

// ---------------------------------------------------------------- hessian --
// H[i][j] = (2/T) sum_t x[t][i] x[t][j]; 64 x 64 tiles, 256 threads, each a
// 4 x 4 block of outputs; t in chunks of 16 through shared memory (fp64).
constexpr int kHT = 64;
constexpr int kHC = 16;

__global__ void __launch_bounds__(256) gptq_hessian_kernel(const __half* __restrict__ X, int64_t T,
                                                           int64_t K, double* __restrict__ H) {
    __shared__ double xi[kHC][kHT];
    __shared__ double xj[kHC][kHT];
    const int64_t i0 = static_cast<int64_t>(blockIdx.y) * kHT;
    const int64_t j0 = static_cast<int64_t>(blockIdx.x) * kHT;
    const int tx = threadIdx.x & 15;   // 4 columns each
    const int ty = threadIdx.x >> 4;   // 4 rows each
    double acc[4][4] = {};
    for (int64_t t0 = 0; t0 < T; t0 += kHC) {
        for (int e = threadIdx.x; e < kHC * kHT; e += 256) {
            const int tt = e / kHT, c = e - tt * kHT;
            const int64_t t = t0 + tt;
            xi[tt][c] = (t < T && i0 + c < K) ? static_cast<double>(__half2float(X[t * K + i0 + c])) : 0.0;
            xj[tt][c] = (t < T && j0 + c < K) ? static_cast<double>(__half2float(X[t * K + j0 + c])) : 0.0;
        }
        __syncthreads();
#pragma unroll 4
        for (int tt = 0; tt < kHC; ++tt) {
            double a[4], b[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) a[r] = xi[tt][4 * ty + r];
#pragma unroll
            for (int c = 0; c < 4; ++c) b[c] = xj[tt][4 * tx + c];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] = fma(a[r], b[c], acc[r][c]);
        }
        __syncthreads();
    }
    const double f = 2.0 / static_cast<double>(T);
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int64_t i = i0 + 4 * ty + r, j = j0 + 4 * tx + c;
            if (i < K && j < K) H[i * K + j] = acc[r][c] * f;
        }
}

// ----------------------------------------------------------------- factor --
// Dead inputs and damping, one CTA: the diagonal's mean after dead entries
// are set to 1, summed in a fixed order.
__global__ void __launch_bounds__(1024) gptq_damp_kernel(double* __restrict__ H, int64_t K, double damp,
                                                         uint8_t* __restrict__ dead) {
    __shared__ double part[1024];
    double s = 0.0;
    for (int64_t j = threadIdx.x; j < K; j += 1024) {
        double h = H[j * K + j];
        const bool d = h == 0.0;
        if (d) h = 1.0;
        dead[j] = d ? 1 : 0;
        H[j * K + j] = h;
        s += h;
    }
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = 512; w > 0; w >>= 1) {
        if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    const double lam = damp * (part[0] / static_cast<double>(K));
    for (int64_t j = threadIdx.x; j < K; j += 1024) H[j * K + j] += lam;
}

// A = P H P (index order reversed), lower triangle.
__global__ void gptq_flip_kernel(const double* __restrict__ H, int64_t K, double* __restrict__ A) {
    const int64_t n = K * K;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = e / K, c = e - r * K;
        if (c <= r) A[e] = H[(K - 1 - r) * K + (K - 1 - c)];
    }
}

// Right-looking Cholesky step j (lower triangle of A, unnormalised columns):
// A[r][c] -= A[r][j] * A[c][j] / A[j][j] for j < c <= r.  Column j and
// everything left of it are final at this step and only read.  2-D grid over
// the trailing square (x = column, contiguous in memory); tiles wholly above
// the diagonal return at once.
__global__ void __launch_bounds__(256) gptq_chol_step_kernel(double* __restrict__ A, int64_t K, int64_t j) {
    const int64_t c = j + 1 + static_cast<int64_t>(blockIdx.x) * 32 + threadIdx.x;
    const int64_t r = j + 1 + static_cast<int64_t>(blockIdx.y) * 8 + threadIdx.y;
    if (static_cast<int64_t>(blockIdx.x) * 32 > static_cast<int64_t>(blockIdx.y) * 8 + 7) return;
    if (r >= K || c > r) return;
    const double inv = 1.0 / A[j * K + j];
    A[r * K + c] -= A[r * K + j] * A[c * K + j] * inv;
}

// Pivots: d[j] = sqrt(A[j][j]) after the last step.
__global__ void gptq_pivot_kernel(const double* __restrict__ A, int64_t K, double* __restrict__ d) {
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < K;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x)
        d[j] = sqrt(A[j * K + j]);
}

// L[r][c] = A[r][c] / d[c] for c <= r (so L[c][c] = d[c]).
__global__ void gptq_chol_scale_kernel(double* __restrict__ A, int64_t K, const double* __restrict__ d) {
    const int64_t n = K * K;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = e / K, c = e - r * K;
        if (c <= r) A[e] = A[e] / d[c];
    }
}

// Z = L^-1 (lower), one warp per column c, stored transposed (Zt[c][i] =
// Z[i][c], so a column is contiguous): forward substitution down the column,
// z_c = 1 / L[c][c], z_i = -(sum_{k=c}^{i-1} L[i][k] z_k) / L[i][i]; each
// lane sums a fixed stride of k, then a fixed shuffle tree adds the lanes.
__global__ void __launch_bounds__(256) gptq_trinv_kernel(const double* __restrict__ L,
                                                         const double* __restrict__ d, int64_t K,
                                                         double* __restrict__ Zt) {
    const int lane = threadIdx.x & 31;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (c >= K) return;
    double* z = Zt + c * K;
    for (int64_t i = lane; i < c; i += 32) z[i] = 0.0;
    if (lane == 0) z[c] = 1.0 / d[c];
    __syncwarp();
    for (int64_t i = c + 1; i < K; ++i) {
        double acc = 0.0;
        const double* li = L + i * K;
        for (int64_t k = c + lane; k < i; k += 32) acc = fma(li[k], z[k], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) z[i] = -acc / d[i];
        __syncwarp();
    }
}

// U[i][j] = fp32(Z[K-1-i][K-1-j]) = fp32(Zt[K-1-j][K-1-i]) for j >= i, 0 below.
__global__ void gptq_u_kernel(const double* __restrict__ Zt, int64_t K, float* __restrict__ U) {
    const int64_t n = K * K;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = e / K, j = e - i * K;
        U[e] = j >= i ? static_cast<float>(Zt[(K - 1 - j) * K + (K - 1 - i)]) : 0.0f;
    }
}

// -------------------------------------------------------------- quantize --
constexpr int kGB = 128;   // columns per block of the column loop

// Dead inputs: zero their weights before the loop.
__global__ void gptq_zero_dead_kernel(float* __restrict__ W, int64_t N, int64_t K,
                                      const uint8_t* __restrict__ dead) {
    const int64_t n = N * K;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x)
        if (dead[e % K]) W[e] = 0.0f;
}

// The block [b, b + 128) of every row: one warp per row, lane l holds columns
// b + 4l .. b + 4l + 3.  Writes codes, scales, the block's errors E[n][0..128)
// and the compensated weights of the block's columns.
template <int BITS>
__global__ void __launch_bounds__(256) gptq_block_kernel(float* __restrict__ W, int64_t N, int64_t K,
                                                         int64_t b, const float* __restrict__ U,
                                                         uint8_t* __restrict__ codes,
                                                         uint16_t* __restrict__ scales,
                                                         float* __restrict__ E,
                                                         int* __restrict__ dev_status) {
    constexpr int kQmax = BITS == 4 ? 7 : 127;
    extern __shared__ __align__(16) float gptq_smem[];
    float (*us)[kGB + 4] = reinterpret_cast<float (*)[kGB + 4]>(gptq_smem);   // U[b + j][b + k]
    const int64_t G = K / 64;
    const int ncol = static_cast<int>(K - b < kGB ? K - b : kGB);   // 64 or 128
    for (int e = threadIdx.x; e < kGB * kGB; e += blockDim.x) {
        const int j = e / kGB, k = e - j * kGB;
        us[j][k] = (j < ncol && k < ncol) ? U[(b + j) * K + b + k] : 0.0f;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (n >= N) return;
    float w[4];
    const bool mine = 4 * lane < ncol;
#pragma unroll
    for (int e = 0; e < 4; ++e) w[e] = mine ? W[n * K + b + 4 * lane + e] : 0.0f;
    float wq[4] = {w[0], w[1], w[2], w[3]};        // the weight each column is quantized from
    int c[4] = {0, 0, 0, 0};
    float sf = 0.0f;
    bool usable = true;
    int status = 0;
    for (int j = 0; j < ncol; ++j) {
        if ((j & 63) == 0) {
            // the group's scale from its current weights: lanes 16g .. 16g+15
            const int g = j >> 6;
            float a = 0.0f;
            bool fin = true;
            if ((lane >> 4) == g) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    a = fmaxf(a, fabsf(w[e]));
                    fin = fin && isfinite(w[e]);
                }
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
            const unsigned bad = __ballot_sync(0xffffffffu, !fin);
            a = __shfl_sync(0xffffffffu, a, 16 * g);
            uint16_t s_bits;
            if (bad != 0) {
                s_bits = 0x7E00u;
                usable = false;
                status = 5;
            } else {
                s_bits = __half_as_ushort(__float2half_rn(__fdiv_rn(a, static_cast<float>(kQmax))));
                usable = s_bits != 0x7C00u;
                if (!usable && status == 0) status = 6;
            }
            sf = usable ? __half2float(__ushort_as_half(s_bits)) : 0.0f;
            if (lane == 0) scales[n * G + (b >> 6) + g] = s_bits;
        }
        // column j: its owner lane takes the code and the error
        const int o = j >> 2, oe = j & 3;
        float err = 0.0f;
        if (lane == o) {
            float wj = w[0];
#pragma unroll
            for (int e = 1; e < 4; ++e)
                if (e == oe) wj = w[e];
            int cj = 0;
            if (usable) {
                if (sf != 0.0f)
                    cj = max(-kQmax, min(kQmax, __float2int_rn(__fdiv_rn(wj, sf))));
                const float dq = __fmul_rn(static_cast<float>(cj), sf);
                err = __fdiv_rn(__fsub_rn(wj, dq), us[j][j]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (e == oe) {
                    c[e] = cj;
                    wq[e] = wj;
                }
        }
        err = __shfl_sync(0xffffffffu, err, o);
        if (lane == 0) E[n * kGB + j] = err;
        // spread over the block's later columns
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int k = 4 * lane + e;
            if (k > j && k < ncol) w[e] = __fmaf_rn(-err, us[j][k], w[e]);
        }
    }
    if (mine) {
#pragma unroll
        for (int e = 0; e < 4; ++e) W[n * K + b + 4 * lane + e] = wq[e];
        if (BITS == 4) {
            const uint16_t p = static_cast<uint16_t>((c[0] & 0xF) | ((c[1] & 0xF) << 4) |
                                                     ((c[2] & 0xF) << 8) | ((c[3] & 0xF) << 12));
            *reinterpret_cast<uint16_t*>(codes + n * (K / 2) + (b + 4 * lane) / 2) = p;
        } else {
            const uint32_t p = (c[0] & 0xFF) | ((c[1] & 0xFF) << 8) | ((c[2] & 0xFF) << 16) |
                               (static_cast<uint32_t>(c[3] & 0xFF) << 24);
            *reinterpret_cast<uint32_t*>(codes + n * K + b + 4 * lane) = p;
        }
    }
    if (lane == 0 && status != 0 && dev_status != nullptr) {
        if (status == 5) atomicExch(dev_status, 5);
        else atomicCAS(dev_status, 0, 6);
    }
}

// The block's errors applied to every later column k >= b + 128:
// W[n][k] = fmaf(-E[n][j], U[b + j][k], W[n][k]) for j = 0 .. 127 in order.
// 64 x 64 output tiles, 256 threads, 4 x 4 each.
constexpr int kTT = 64;
__global__ void __launch_bounds__(256) gptq_trail_kernel(float* __restrict__ W, int64_t N, int64_t K,
                                                         int64_t b, const float* __restrict__ U,
                                                         const float* __restrict__ E) {
    extern __shared__ __align__(16) float gptq_smem[];
    float (*es)[kTT] = reinterpret_cast<float (*)[kTT]>(gptq_smem);                 // E[n0 + r][j] as es[j][r]
    float (*ust)[kTT] = reinterpret_cast<float (*)[kTT]>(gptq_smem + kGB * kTT);   // U[b + j][k0 + c]
    const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kTT;
    const int64_t k0 = b + kGB + static_cast<int64_t>(blockIdx.x) * kTT;
    for (int e = threadIdx.x; e < kGB * kTT; e += 256) {
        const int r = e / kGB, j = e - r * kGB;            // coalesced along j of E
        es[j][r] = (n0 + r < N) ? E[(n0 + r) * kGB + j] : 0.0f;
        const int jj = e / kTT, cc = e - jj * kTT;        // coalesced along k of U
        ust[jj][cc] = (k0 + cc < K) ? U[(b + jj) * K + k0 + cc] : 0.0f;
    }
    __syncthreads();
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float w[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const int64_t n = n0 + 4 * ty + r, k = k0 + 4 * tx + cc;
            w[r][cc] = (n < N && k < K) ? W[n * K + k] : 0.0f;
        }
#pragma unroll 4
    for (int j = 0; j < kGB; ++j) {
        const float4 ev = *reinterpret_cast<const float4*>(&es[j][4 * ty]);
        const float4 uv = *reinterpret_cast<const float4*>(&ust[j][4 * tx]);
        const float e4[4] = {ev.x, ev.y, ev.z, ev.w};
        const float u4[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) w[r][cc] = __fmaf_rn(-e4[r], u4[cc], w[r][cc]);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const int64_t n = n0 + 4 * ty + r, k = k0 + 4 * tx + cc;
            if (n < N && k < K) W[n * K + k] = w[r][cc];
        }
}

// ---------------------------------------------------------------- launchers --
static int grid_for(int64_t n, int threads) {
    int64_t g = (n + threads - 1) / threads;
    if (g > 148LL * 32) g = 148LL * 32;
    return static_cast<int>(g < 1 ? 1 : g);
}

cudaError_t launch_gptq_hessian(const uint16_t* X, int64_t T, int64_t K, double* H, cudaStream_t s) {
    const dim3 grid(static_cast<unsigned>((K + kHT - 1) / kHT), static_cast<unsigned>((K + kHT - 1) / kHT));
    gptq_hessian_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const __half*>(X), T, K, H);
    return cudaGetLastError();
}

// work: K * K + K doubles.  H is consumed (it ends up holding L^-1, transposed).
cudaError_t launch_gptq_factor(double* H, int64_t K, double damp, float* U, uint8_t* dead,
                               double* work, cudaStream_t s) {
    gptq_damp_kernel<<<1, 1024, 0, s>>>(H, K, damp, dead);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    double* A = work;              // P H P, factored in place
    double* d = work + K * K;      // pivots
    gptq_flip_kernel<<<grid_for(K * K, 256), 256, 0, s>>>(H, K, A);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    for (int64_t j = 0; j + 1 < K; ++j) {
        const int64_t m = K - 1 - j;
        const dim3 grid(static_cast<unsigned>((m + 31) / 32), static_cast<unsigned>((m + 7) / 8));
        gptq_chol_step_kernel<<<grid, dim3(32, 8), 0, s>>>(A, K, j);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    gptq_pivot_kernel<<<grid_for(K, 256), 256, 0, s>>>(A, K, d);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    gptq_chol_scale_kernel<<<grid_for(K * K, 256), 256, 0, s>>>(A, K, d);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    gptq_trinv_kernel<<<static_cast<unsigned>((K + 7) / 8), 256, 0, s>>>(A, d, K, H);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    gptq_u_kernel<<<grid_for(K * K, 256), 256, 0, s>>>(H, K, U);
    return cudaGetLastError();
}

// W: fp32 [N, K] in/out; work: fp32 [N, 128] (the errors of one block).
cudaError_t launch_gptq_quantize(float* W, int64_t N, int64_t K, int bits, const float* U,
                                 const uint8_t* dead, void* codes, uint16_t* scales, float* work,
                                 int* dev_status, cudaStream_t s) {
    cudaError_t e;
    if (dead != nullptr) {
        gptq_zero_dead_kernel<<<grid_for(N * K, 256), 256, 0, s>>>(W, N, K, dead);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const unsigned rows_grid = static_cast<unsigned>((N + 7) / 8);
    constexpr int kBlockSmem = kGB * (kGB + 4) * 4;
    constexpr int kTrailSmem = 2 * kGB * kTT * 4;
    static bool attr_set[64] = {};
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        if ((e = cudaFuncSetAttribute(gptq_block_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kBlockSmem)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(gptq_block_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kBlockSmem)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(gptq_trail_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kTrailSmem)) != cudaSuccess)
            return e;
        attr_set[dev] = true;
    }
    for (int64_t b = 0; b < K; b += kGB) {
        if (bits == 4)
            gptq_block_kernel<4><<<rows_grid, 256, kBlockSmem, s>>>(W, N, K, b, U, static_cast<uint8_t*>(codes),
                                                           scales, work, dev_status);
        else
            gptq_block_kernel<8><<<rows_grid, 256, kBlockSmem, s>>>(W, N, K, b, U, static_cast<uint8_t*>(codes),
                                                           scales, work, dev_status);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t rest = K - b - kGB;
        if (rest > 0) {
            const dim3 grid(static_cast<unsigned>((rest + kTT - 1) / kTT),
                            static_cast<unsigned>((N + kTT - 1) / kTT));
            gptq_trail_kernel<<<grid, 256, kTrailSmem, s>>>(W, N, K, b, U, work);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

}  // namespace rq
