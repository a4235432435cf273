// codec_fit.cu -- SVD initialisation of the cross-loop codec on the GPU.
//
// "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers", review
// page, "What carries the argument": the codec starts from the top right singular vectors
// of the centred teacher activations.  For every (layer, stored head, axis) group and its
// n calibration vectors x_i (width W = T * Dp, loop-major):
//   mu = (1/n) sum_i x_i,   Y = X - mu,   Y = U diag(sigma) V^T,
//   W_down = V[:, :r] (each column signed so its largest-magnitude entry is positive),
//   W_up,t = transpose of the loop-t row block of W_down,  mu_t = loop-t slice of mu.
// The calibration set is small (n of a few hundred) while W is T*d or T*H*d, so the
// eigenproblem is solved on the dual Gram matrix K = Y Y^T (n x n) and the right vectors
// are recovered as v_j = Y^T u_j / sigma_j.  All arithmetic is fp64 (the Gram matrix
// squares the spread of the singular values).
//
// Kernels (one launch each, every group in one grid):
//   fit_mean     mu per column
//   fit_gram     K = Y Y^T, 32 x 32 tiles staged in shared memory
//   fit_jacobi   parallel cyclic Jacobi on K (one CTA per group): in each round the n
//                indices form n/2 disjoint pairs (round-robin "circle" order), every pair
//                gets the rotation that zeroes its off-diagonal entry, and K <- J^T K J,
//                U <- U J are applied as independent 2 x 2 blocks; sweeps of n-1 rounds
//                until a sweep finds nothing left to rotate
//   fit_order    eigenvalues sorted descending, sigma = sqrt(lambda)
//   fit_vectors  v_j = Y^T u_j / sigma_j for the r leading pairs
//   fit_finish   sign convention, bf16/fp32 stores of W_down and W_up
#include "encode.cuh"

namespace lla {
namespace {

constexpr int kFitMaxSweeps = 40;
constexpr int kJacobiThreads = 512;
constexpr int kJacobiUnroll = 4; // blocks / entries per thread and pass (loads first)

struct FitArgs {
    const void *x;          // T [n_layers][n][T][H][d] (one axis)
    int64_t n;
    int32_t T, H, d, Dp, Hs, W, fold, r, layer0;
    double *mu64;           // [G][W]
    double *K;              // [G][n][n]
    double *U;              // [G][n][n]
    double *lam;            // [G][n] eigenvalues, descending
    int32_t *order;         // [G][n] index of the j-th largest eigenvalue
    double *V;              // [G][r][W]
    int32_t *status;        // sticky: LLA_ERR_NO_CONVERGENCE; status[1] += sweeps of every group
    void *W_down;           // T [L][H'][r][W]
    float *W_up;            // [L][H'][T][r][Dp]
    float *mu;              // [L][H'][T][Dp]
    float *sigma;           // [n_layers][H'][n] or null
};

template <typename T> __device__ __forceinline__ double ld_x(const FitArgs &a, int g, int64_t i, int c)
{
    const int l = g / a.Hs, hs = g - l * a.Hs;
    const int t = c / a.Dp, k = c - t * a.Dp;
    const int64_t off = (((int64_t)l * a.n + i) * a.T + t) * a.H * a.d + (a.fold ? 0 : hs * a.d) + k;
    return (double)Elem<T>::to_f(static_cast<const T *>(a.x)[off]);
}

template <typename T> __global__ void __launch_bounds__(128) fit_mean_kernel(const FitArgs a)
{
    const int g = blockIdx.y;
    const int c = blockIdx.x * 128 + threadIdx.x;
    if (c >= a.W)
        return;
    double s = 0.0;
    for (int64_t i = 0; i < a.n; ++i)
        s += ld_x<T>(a, g, i, c);
    const double m = s / (double)a.n;
    a.mu64[(int64_t)g * a.W + c] = m;
    const int l = g / a.Hs, hs = g - l * a.Hs;
    a.mu[((int64_t)(a.layer0 + l) * a.Hs + hs) * a.W + c] = (float)m;
}

// K tile (32 x 32) of group g; 256 threads, 2 x 2 outputs each.
template <typename T> __global__ void __launch_bounds__(256) fit_gram_kernel(const FitArgs a)
{
    __shared__ double yi[32][33], yj[32][33];
    const int g = blockIdx.z;
    const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const double *mu = a.mu64 + (int64_t)g * a.W;
    double acc[2][2] = {{0.0, 0.0}, {0.0, 0.0}};
    for (int c0 = 0; c0 < a.W; c0 += 32) {
        for (int e = threadIdx.x; e < 32 * 32; e += 256) {
            const int row = e >> 5, col = e & 31;
            const int c = c0 + col;
            double vi = 0.0, vj = 0.0;
            if (c < a.W) {
                if (i0 + row < a.n)
                    vi = ld_x<T>(a, g, i0 + row, c) - mu[c];
                if (j0 + row < a.n)
                    vj = ld_x<T>(a, g, j0 + row, c) - mu[c];
            }
            yi[row][col] = vi;
            yj[row][col] = vj;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const double a0 = yi[2 * ty][k], a1 = yi[2 * ty + 1][k];
            const double b0 = yj[2 * tx][k], b1 = yj[2 * tx + 1][k];
            acc[0][0] = fma(a0, b0, acc[0][0]);
            acc[0][1] = fma(a0, b1, acc[0][1]);
            acc[1][0] = fma(a1, b0, acc[1][0]);
            acc[1][1] = fma(a1, b1, acc[1][1]);
        }
        __syncthreads();
    }
    double *K = a.K + (int64_t)g * a.n * a.n;
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int v = 0; v < 2; ++v) {
            const int64_t i = i0 + 2 * ty + u, j = j0 + 2 * tx + v;
            if (i < a.n && j < a.n)
                K[i * a.n + j] = acc[u][v];
        }
}

// Parallel cyclic Jacobi on the symmetric K of one group (n even, n <= 2 * kJacobiThreads).
__global__ void __launch_bounds__(kJacobiThreads) fit_jacobi_kernel(const FitArgs a)
{
    __shared__ int P[kJacobiThreads], Q[kJacobiThreads];
    __shared__ double cs[kJacobiThreads], sn[kJacobiThreads];
    __shared__ int rotated;
    __shared__ double floor_abs;
    const int g = blockIdx.x;
    const int n = (int)a.n, np = n / 2;
    double *K = a.K + (int64_t)g * n * n;
    double *U = a.U + (int64_t)g * n * n;
    for (int64_t e = threadIdx.x; e < (int64_t)n * n; e += blockDim.x)
        U[e] = (e / n == e % n) ? 1.0 : 0.0;
    if (threadIdx.x == 0) {
        // an absolute floor for the off-diagonal entries, invariant under the rotations:
        // centred data make K singular, and the relative test alone would keep rotating
        // rounding noise against the null direction
        double tr = 0.0;
        for (int i = 0; i < n; ++i)
            tr += K[(int64_t)i * n + i];
        floor_abs = 1e-14 * tr;
    }
    __syncthreads();
    bool converged = false;
    int sweeps = 0;
    for (int sweep = 0; sweep < kFitMaxSweeps && !converged; ++sweep, ++sweeps) {
        if (threadIdx.x == 0)
            rotated = 0;
        __syncthreads();
        for (int round = 0; round < n - 1; ++round) {
            // circle order: position 0 fixed, positions 1..n-1 rotate by `round`
            for (int k = threadIdx.x; k < np; k += blockDim.x) {
                auto at = [&](int pos) { return pos == 0 ? 0 : ((pos - 1 + round) % (n - 1)) + 1; };
                const int p = at(k), q = at(n - 1 - k);
                const double app = K[(int64_t)p * n + p], aqq = K[(int64_t)q * n + q], apq = K[(int64_t)p * n + q];
                double c = 1.0, s = 0.0;
                if (fabs(apq) > fmax(1e-15 * sqrt(fabs(app * aqq)), floor_abs)) {
                    // the rotation J = [[c, s], [-s, c]] with (J^T A J)_pq = 0 (symmetric Schur)
                    const double tau = (aqq - app) / (2.0 * apq);
                    const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
                    c = 1.0 / sqrt(1.0 + t * t);
                    s = t * c;
                    rotated = 1; // benign race: every writer stores 1
                }
                P[k] = p;
                Q[k] = q;
                cs[k] = c;
                sn[k] = s;
            }
            __syncthreads();
            // K <- J^T K J, one 2 x 2 block (pair a rows, pair b columns) per step;
            // kJacobiUnroll blocks per thread and pass, all loads issued before the stores (the
            // blocks are disjoint, but the compiler cannot know it)
            const int64_t nblk = (int64_t)np * np;
            for (int64_t e0 = threadIdx.x; e0 < nblk; e0 += kJacobiUnroll * (int64_t)blockDim.x) {
                double m[kJacobiUnroll][4];
                int r0i[kJacobiUnroll], r1i[kJacobiUnroll], c0i[kJacobiUnroll], c1i[kJacobiUnroll], pi[kJacobiUnroll],
                    pj[kJacobiUnroll];
                bool ok[kJacobiUnroll];
#pragma unroll
                for (int u = 0; u < kJacobiUnroll; ++u) {
                    const int64_t e = e0 + (int64_t)u * blockDim.x;
                    ok[u] = e < nblk;
                    const int ia = ok[u] ? (int)(e / np) : 0, ib = ok[u] ? (int)(e - (int64_t)ia * np) : 0;
                    pi[u] = ia;
                    pj[u] = ib;
                    r0i[u] = P[ia];
                    r1i[u] = Q[ia];
                    c0i[u] = P[ib];
                    c1i[u] = Q[ib];
                    if (ok[u]) {
                        m[u][0] = K[(int64_t)r0i[u] * n + c0i[u]];
                        m[u][1] = K[(int64_t)r0i[u] * n + c1i[u]];
                        m[u][2] = K[(int64_t)r1i[u] * n + c0i[u]];
                        m[u][3] = K[(int64_t)r1i[u] * n + c1i[u]];
                    }
                }
#pragma unroll
                for (int u = 0; u < kJacobiUnroll; ++u) {
                    if (!ok[u])
                        continue;
                    const double ca = cs[pi[u]], sa = sn[pi[u]], cb = cs[pj[u]], sb = sn[pj[u]];
                    const double t00 = m[u][0] * cb - m[u][1] * sb, t01 = m[u][0] * sb + m[u][1] * cb;
                    const double t10 = m[u][2] * cb - m[u][3] * sb, t11 = m[u][2] * sb + m[u][3] * cb;
                    K[(int64_t)r0i[u] * n + c0i[u]] = ca * t00 - sa * t10;
                    K[(int64_t)r0i[u] * n + c1i[u]] = ca * t01 - sa * t11;
                    K[(int64_t)r1i[u] * n + c0i[u]] = sa * t00 + ca * t10;
                    K[(int64_t)r1i[u] * n + c1i[u]] = sa * t01 + ca * t11;
                }
            }
            // U <- U J, kJacobiUnroll (row, pair) entries per thread and pass
            const int64_t nup = (int64_t)n * np;
            for (int64_t e0 = threadIdx.x; e0 < nup; e0 += kJacobiUnroll * (int64_t)blockDim.x) {
                double up[kJacobiUnroll], uq[kJacobiUnroll];
                int64_t ip[kJacobiUnroll], iq[kJacobiUnroll];
                int kk[kJacobiUnroll];
                bool ok[kJacobiUnroll];
#pragma unroll
                for (int u = 0; u < kJacobiUnroll; ++u) {
                    const int64_t e = e0 + (int64_t)u * blockDim.x;
                    ok[u] = e < nup;
                    const int row = ok[u] ? (int)(e / np) : 0, k = ok[u] ? (int)(e - (int64_t)row * np) : 0;
                    kk[u] = k;
                    ip[u] = (int64_t)row * n + P[k];
                    iq[u] = (int64_t)row * n + Q[k];
                    if (ok[u]) {
                        up[u] = U[ip[u]];
                        uq[u] = U[iq[u]];
                    }
                }
#pragma unroll
                for (int u = 0; u < kJacobiUnroll; ++u) {
                    if (!ok[u])
                        continue;
                    U[ip[u]] = cs[kk[u]] * up[u] - sn[kk[u]] * uq[u];
                    U[iq[u]] = sn[kk[u]] * up[u] + cs[kk[u]] * uq[u];
                }
            }
            __syncthreads();
        }
        converged = rotated == 0;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        atomicAdd(a.status + 1, sweeps);
        if (!converged)
            report_status(a.status, LLA_ERR_NO_CONVERGENCE);
    }
}

// Eigenvalues of K (its diagonal after Jacobi) ranked descending; sigma = sqrt(lambda).
__global__ void __launch_bounds__(256) fit_order_kernel(const FitArgs a)
{
    const int g = blockIdx.x;
    const int n = (int)a.n;
    const double *K = a.K + (int64_t)g * n * n;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const double li = K[(int64_t)i * n + i];
        int rank = 0;
        for (int j = 0; j < n; ++j) {
            const double lj = K[(int64_t)j * n + j];
            rank += (lj > li || (lj == li && j < i)) ? 1 : 0;
        }
        a.order[(int64_t)g * n + rank] = i;
        a.lam[(int64_t)g * n + rank] = li;
        if (a.sigma != nullptr)
            a.sigma[(int64_t)g * n + rank] = (float)sqrt(fmax(li, 0.0));
    }
}

// v_j[c] = sum_i y_i[c] u_i,order[j] / sigma_j for the r leading pairs.
template <typename T> __global__ void __launch_bounds__(128) fit_vectors_kernel(const FitArgs a)
{
    const int g = blockIdx.z, j = blockIdx.y;
    const int c = blockIdx.x * 128 + threadIdx.x;
    if (c >= a.W)
        return;
    const int n = (int)a.n;
    const int oj = a.order[(int64_t)g * n + j];
    const double sig = sqrt(fmax(a.lam[(int64_t)g * n + j], 0.0));
    const double *U = a.U + (int64_t)g * n * n;
    const double m = a.mu64[(int64_t)g * a.W + c];
    double s = 0.0;
    for (int i = 0; i < n; ++i)
        s = fma(ld_x<T>(a, g, i, c) - m, U[(int64_t)i * n + oj], s);
    a.V[((int64_t)g * a.r + j) * a.W + c] = sig > 0.0 ? s / sig : 0.0;
}

// Sign convention (largest-magnitude entry positive, first one on a tie) and the stores.
template <typename T> __global__ void __launch_bounds__(256) fit_finish_kernel(const FitArgs a)
{
    __shared__ double best_v[256];
    __shared__ int best_c[256];
    const int g = blockIdx.y, j = blockIdx.x;
    const double *v = a.V + ((int64_t)g * a.r + j) * a.W;
    double bv = -1.0;
    int bc = 0x7fffffff;
    for (int c = threadIdx.x; c < a.W; c += blockDim.x) {
        const double m = fabs(v[c]);
        if (m > bv || (m == bv && c < bc)) {
            bv = m;
            bc = c;
        }
    }
    best_v[threadIdx.x] = bv;
    best_c[threadIdx.x] = bc;
    __syncthreads();
    for (int off = blockDim.x / 2; off > 0; off >>= 1) {
        if (threadIdx.x < off) {
            const double ov = best_v[threadIdx.x + off];
            const int oc = best_c[threadIdx.x + off];
            if (ov > best_v[threadIdx.x] || (ov == best_v[threadIdx.x] && oc < best_c[threadIdx.x])) {
                best_v[threadIdx.x] = ov;
                best_c[threadIdx.x] = oc;
            }
        }
        __syncthreads();
    }
    const double sign = v[best_c[0]] < 0.0 ? -1.0 : 1.0;
    const int l = g / a.Hs, hs = g - l * a.Hs;
    const int64_t grp = (int64_t)(a.layer0 + l) * a.Hs + hs;
    T *wd = static_cast<T *>(a.W_down) + (grp * a.r + j) * a.W;
    float *wu = a.W_up + grp * a.T * a.r * a.Dp;
    for (int c = threadIdx.x; c < a.W; c += blockDim.x) {
        const double x = sign * v[c];
        wd[c] = Elem<T>::from_f((float)x);
        const int t = c / a.Dp, k = c - t * a.Dp;
        wu[((int64_t)t * a.r + j) * a.Dp + k] = (float)x;
    }
}

template <typename T> cudaError_t run_fit(const FitArgs &a, int groups, cudaStream_t stream)
{
    const unsigned cw = (unsigned)((a.W + 127) / 128), nt = (unsigned)((a.n + 31) / 32);
    fit_mean_kernel<T><<<dim3(cw, groups), 128, 0, stream>>>(a);
    fit_gram_kernel<T><<<dim3(nt, nt, groups), 256, 0, stream>>>(a);
    fit_jacobi_kernel<<<groups, kJacobiThreads, 0, stream>>>(a);
    fit_order_kernel<<<groups, 256, 0, stream>>>(a);
    fit_vectors_kernel<T><<<dim3(cw, a.r, groups), 128, 0, stream>>>(a);
    fit_finish_kernel<T><<<dim3(a.r, groups), 256, 0, stream>>>(a);
    return cudaGetLastError();
}

} // namespace

size_t codec_fit_scratch_bytes(int64_t groups, int64_t n, int64_t W, int64_t r_max)
{
    const size_t per = sizeof(double) * (size_t)(W + 2 * n * n + n + r_max * W) + sizeof(int32_t) * (size_t)n;
    return (size_t)groups * ((per + 255) & ~(size_t)255);
}

cudaError_t launch_codec_fit(const CodecFitArgs &c, cudaStream_t stream)
{
    const int64_t G = (int64_t)c.n_layers * c.Hs;
    if (G > 65535 || c.n > 2 * kJacobiThreads || (c.n & 1))
        return cudaErrorInvalidValue;
    const int r_max = c.r_k > c.r_v ? c.r_k : c.r_v;
    uint8_t *ws = static_cast<uint8_t *>(c.scratch);
    for (int axis = 0; axis < 2; ++axis) {
        FitArgs a;
        a.x = axis ? c.x_v : c.x_k;
        a.n = c.n;
        a.T = c.T; a.H = c.H; a.d = c.d; a.Dp = c.Dp; a.Hs = c.Hs; a.W = c.W; a.fold = c.fold;
        a.r = axis ? c.r_v : c.r_k;
        a.layer0 = c.layer0;
        // carve the scratch by region (the axes run one after the other and share it)
        size_t off = 0;
        auto take = [&](size_t bytes) { uint8_t *p = ws + off; off += (bytes + 255) & ~(size_t)255; return p; };
        a.mu64 = reinterpret_cast<double *>(take(sizeof(double) * G * c.W));
        a.K = reinterpret_cast<double *>(take(sizeof(double) * G * c.n * c.n));
        a.U = reinterpret_cast<double *>(take(sizeof(double) * G * c.n * c.n));
        a.lam = reinterpret_cast<double *>(take(sizeof(double) * G * c.n));
        a.order = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * G * c.n));
        a.V = reinterpret_cast<double *>(take(sizeof(double) * G * r_max * c.W));
        a.status = c.status;
        a.W_down = axis ? c.W_down_v : c.W_down_k;
        a.W_up = axis ? c.W_up_v : c.W_up_k;
        a.mu = axis ? c.mu_v : c.mu_k;
        a.sigma = axis ? c.sigma_v : c.sigma_k;
        const cudaError_t e = c.dtype == LLA_BF16 ? run_fit<__nv_bfloat16>(a, (int)G, stream)
                                                  : run_fit<float>(a, (int)G, stream);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

} // namespace lla
