// Codec fit on the GPU: the SVD initialisation of W_down from calibration stacks.
//
// [LLA §3, "Initialisation and conversion"]: for each (layer, head, axis) the calibration
// stacks X (n x S, S = T*d_head; the 2D variant stacks the heads too) are centred with their
// mean mu, and W_down is the top-r right singular vectors of X - mu; loop t's up-projection is
// the loop-t row slice of W_down.  This file computes mu, W_down and the top-r singular values
// for P independent problems at once, in fp64 throughout:
//
//   1. mu = column means of X.
//   2. The Gram matrix of the smaller side, m = min(n, S):  G = Xcᵀ Xc (S x S) when S <= n,
//      else G = Xc Xcᵀ (n x n); its top-r eigenvectors are the right (resp. left) singular
//      vectors, eigenvalues sigma².
//   3. Subspace iteration on G with a block of k = min(m, max(2r, r + 16)) columns, started
//      from a fixed pseudo-random block: `iters` products with G, orthonormalised after every
//      second one (Z <- orth(G G Z)).  orth is shifted
//      CholeskyQR3 (Fukaya, Kannan, Nakatsukasa, Yamamoto and Yanagisawa, "Shifted Cholesky QR
//      for computing the QR factorization of ill-conditioned matrices", SIAM J. Sci. Comput.
//      2020): one Cholesky QR pass of Yᵀ Y + s I with s = 11 (m k + k (k + 1)) u ||Y||_F², then
//      two plain passes; each pass forms the k x k Gram, its Cholesky factor L, L⁻¹ and Y L⁻ᵀ.
//   4. Rayleigh–Ritz: H = Zᵀ G Z (k x k), diagonalised by cyclic Jacobi rotations in the
//      round-robin parallel order (Golub & Van Loan, "Matrix Computations", §8.5: the symmetric
//      2x2 Schur decomposition and the parallel ordering); the top r Ritz pairs (by value, ties
//      by index) give W = Z V_r, or for n < S, W = Xcᵀ (Z V_r) normalised per column.
//   5. Each column is flipped so that its entry of largest magnitude (first on ties) is
//      positive, the convention of the FP64 host fit.
//
// The iteration is the approximation: singular values and the fitted subspace converge as
// (lambda_{k+1} / lambda_r)^iters; 24 iterations (the default) reach ~1e-8 relative on the seeded smooth
// stacks (rank-R trajectories plus noise) of the test configurations.  Every kernel is plain CUDA-core
// fp64 (the work is a few GFLOP per problem, dominated by latency of the small factorizations).
#include <math.h>
#include <stdint.h>

#include "lla_internal.cuh"

namespace {

constexpr int kOver = 16;       // subspace block beyond the rank: k = min(m, max(2r, r + kOver))
constexpr int kMaxK = 1024;     // block size limit (one Cholesky column per thread)
constexpr int kJacobiSweeps = 30;
constexpr double kUnit = 1.1102230246251565e-16;  // 2^-53

// ---------------------------------------------------------------------------------------------
// 1. column means
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) fit_mean_kernel(const float* X, int n, int S, double* mu, float* mu_out) {
    const int p = blockIdx.y;
    const int c = blockIdx.x * 256 + threadIdx.x;
    if (c >= S) return;
    const float* x = X + size_t(p) * n * S + c;
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += double(x[size_t(i) * S]);
    const double v = s / n;
    mu[size_t(p) * S + c] = v;
    mu_out[size_t(p) * S + c] = float(v);
}

// ---------------------------------------------------------------------------------------------
// 2. Gram matrix of the centred stacks, 64 x 64 tiles of the lower triangle, mirrored
// ---------------------------------------------------------------------------------------------
// a(l, i): col-Gram (m = S): X[l][i] - mu[i], l < n;  row-Gram (m = n): X[i][l] - mu[l], l < S.
__global__ void __launch_bounds__(256) fit_gram_kernel(const float* X, const double* mu, int n, int S, int m,
                                                       int col, double* G) {
    const int p = blockIdx.y;
    // lower-triangle tile (ti, tj), tj <= ti, from the linear index
    const int x = blockIdx.x;
    int ti = int((sqrt(8.0 * x + 1.0) - 1.0) * 0.5);
    while ((ti + 1) * (ti + 2) / 2 <= x) ++ti;
    while (ti * (ti + 1) / 2 > x) --ti;
    const int tj = x - ti * (ti + 1) / 2;
    const int i0 = ti * 64, j0 = tj * 64;
    const float* Xp = X + size_t(p) * n * S;
    const double* mp = mu + size_t(p) * S;
    const int L = col ? n : S;
    __shared__ double As[16][64], Bs[16][64];
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    double acc[4][4] = {};
    for (int l0 = 0; l0 < L; l0 += 16) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int e = tid + 256 * q;
            int ll, ii;
            if (col) {
                ll = e >> 6;
                ii = e & 63;
            } else {
                ii = e >> 4;
                ll = e & 15;
            }
            const int l = l0 + ll;
            double a = 0.0, b = 0.0;
            if (l < L) {
                const int ia = i0 + ii, ib = j0 + ii;
                if (col) {
                    if (ia < m) a = double(Xp[size_t(l) * S + ia]) - mp[ia];
                    if (ib < m) b = double(Xp[size_t(l) * S + ib]) - mp[ib];
                } else {
                    const double ml = mp[l];
                    if (ia < m) a = double(Xp[size_t(ia) * S + l]) - ml;
                    if (ib < m) b = double(Xp[size_t(ib) * S + l]) - ml;
                }
            }
            As[ll][ii] = a;
            Bs[ll][ii] = b;
        }
        __syncthreads();
#pragma unroll
        for (int ll = 0; ll < 16; ++ll) {
            double a[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                a[u] = As[ll][ty + 16 * u];
                b[u] = Bs[ll][tx + 16 * u];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fma(a[u], b[v], acc[u][v]);
        }
        __syncthreads();
    }
    double* Gp = G + size_t(p) * m * m;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int i = i0 + ty + 16 * u, j = j0 + tx + 16 * v;
            if (i < m && j < m) {
                Gp[size_t(i) * m + j] = acc[u][v];
                Gp[size_t(j) * m + i] = acc[u][v];
            }
        }
}

// ---------------------------------------------------------------------------------------------
// 3. starting block: a fixed counter-based pseudo-random value in [-1, 1) per (problem, i, c)
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint64_t mix64(uint64_t x) {  // the splitmix64 finaliser
    x ^= x >> 30;
    x *= 0xBF58476D1CE4E5B9ull;
    x ^= x >> 27;
    x *= 0x94D049BB133111EBull;
    x ^= x >> 31;
    return x;
}
__global__ void __launch_bounds__(256) fit_init_kernel(double* Z, int m, int k) {
    const int p = blockIdx.y;
    const int e = blockIdx.x * 256 + threadIdx.x;
    if (e >= m * k) return;
    const int i = e / k, c = e - i * k;
    const uint64_t h = mix64(uint64_t(p) * 0x9E3779B97F4A7C15ull + uint64_t(i) * 0xBF58476D1CE4E5B9ull +
                             uint64_t(c) * 0x94D049BB133111EBull + 0x2545F4914F6CDD1Dull);
    Z[size_t(p) * m * k + e] = double(h >> 11) * 0x1.0p-53 * 2.0 - 1.0;
}

// ---------------------------------------------------------------------------------------------
// batched fp64 GEMM C = A B with strided operand access, 64 x 64 tiles, K chunks of 16
// ---------------------------------------------------------------------------------------------
struct DOp {  // element (i, l) of problem p at base + p*batch + i*rs + l*cs
    const double* base;
    long long batch;
    int rs, cs;
    __device__ double operator()(int p, int i, int l) const {
        return base[p * batch + (long long)i * rs + (long long)l * cs];
    }
    __device__ bool l_contiguous() const { return cs == 1; }
};
struct XcT {  // element (i, l) = X[p][l][i] - mu[p][i]: the centred stacks, transposed (S x n)
    const float* X;
    const double* mu;
    int n, S;
    __device__ double operator()(int p, int i, int l) const {
        return double(X[(size_t(p) * n + l) * S + i]) - mu[size_t(p) * S + i];
    }
    __device__ bool l_contiguous() const { return false; }
};

template <class OA>
__global__ void __launch_bounds__(64) fit_gemm_kernel(int M, int N, int K, OA A, DOp B, double* C, long long c_batch,
                                                      int ldc) {
    // 64 x 64 tile, 64 threads, 8 x 8 outputs per thread (rows ty + 8u, columns tx + 8v): one
    // shared-memory load per four FMAs
    const int p = blockIdx.z;
    const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
    __shared__ double As[16][64], Bs[16][64];
    const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
    const bool a_l = A.l_contiguous(), b_l = B.l_contiguous();
    double acc[8][8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[u][v] = 0.0;
    for (int l0 = 0; l0 < K; l0 += 16) {
#pragma unroll 4
        for (int q = 0; q < 16; ++q) {
            const int e = tid + 64 * q;
            int ll = a_l ? (e & 15) : (e >> 6), ii = a_l ? (e >> 4) : (e & 63);
            As[ll][ii] = (i0 + ii < M && l0 + ll < K) ? A(p, i0 + ii, l0 + ll) : 0.0;
            ll = b_l ? (e & 15) : (e >> 6);
            const int jj = b_l ? (e >> 4) : (e & 63);
            Bs[ll][jj] = (j0 + jj < N && l0 + ll < K) ? B(p, l0 + ll, j0 + jj) : 0.0;
        }
        __syncthreads();
#pragma unroll 2
        for (int ll = 0; ll < 16; ++ll) {
            double a[8], b[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                a[u] = As[ll][ty + 8 * u];
                b[u] = Bs[ll][tx + 8 * u];
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int v = 0; v < 8; ++v) acc[u][v] = fma(a[u], b[v], acc[u][v]);
        }
        __syncthreads();
    }
    double* Cp = C + p * c_batch;
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int i = i0 + ty + 8 * u, j = j0 + tx + 8 * v;
            if (i < M && j < N) Cp[size_t(i) * ldc + j] = acc[u][v];
        }
}

// ---------------------------------------------------------------------------------------------
// Cholesky factor (lower, in place) of a k x k Gram, optionally shifted; one CTA per problem
// ---------------------------------------------------------------------------------------------
__device__ double block_sum(double v, double* red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = (blockDim.x + 31) >> 5;
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    double t = 0.0;
    for (int i = 0; i < nw; ++i) t += red[i];
    __syncthreads();
    return t;
}

__global__ void __launch_bounds__(1024) fit_chol_kernel(double* Kg, int k, int m, int shifted, uint32_t* status) {
    // right-looking, one column at a time; the trailing update runs one warp per row
    double* A = Kg + size_t(blockIdx.x) * k * k;
    __shared__ double colj[kMaxK];
    __shared__ double red[32];
    __shared__ double piv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
    if (shifted) {
        double tr = 0.0;
        for (int i = tid; i < k; i += blockDim.x) tr += A[size_t(i) * k + i];
        tr = block_sum(tr, red);
        const double s = 11.0 * (double(m) * k + double(k) * (k + 1)) * kUnit * tr;
        for (int i = tid; i < k; i += blockDim.x) A[size_t(i) * k + i] += s;
        __syncthreads();
    }
    for (int j = 0; j < k; ++j) {
        if (tid == 0) {
            double d = A[size_t(j) * k + j];
            if (!(d > 0.0)) {  // not positive definite: record it, continue on a tiny pivot
                atomicOr(status, LLA_FLAG_FIT_BREAKDOWN);
                d = 1e-300;
            }
            piv = sqrt(d);
            A[size_t(j) * k + j] = piv;
        }
        __syncthreads();
        const double inv = 1.0 / piv;
        for (int i = j + 1 + tid; i < k; i += blockDim.x) {
            const double v = A[size_t(i) * k + j] * inv;
            A[size_t(i) * k + j] = v;
            colj[i] = v;
        }
        __syncthreads();
        for (int i = j + 1 + warp; i < k; i += nw) {  // contiguous row segments, no divisions
            const double ci = colj[i];
            double* row = A + size_t(i) * k;
            for (int l = j + 1 + lane; l <= i; l += 32) row[l] -= ci * colj[l];
        }
        __syncthreads();
    }
}

// L⁻¹ of the lower factor, full k x k output: one warp per column j (forward substitution down
// the column; the lanes split each row's dot product), the column kept in shared memory
__device__ __forceinline__ double warp_sum_d(double v) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__global__ void __launch_bounds__(1024) fit_trinv_kernel(const double* Kg, double* Li, int k) {
    extern __shared__ double trinv_col[];  // [warps][k]
    const int p = blockIdx.y, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x * (blockDim.x >> 5) + w;
    if (j >= k) return;  // whole warps only; no block-wide barrier below
    const double* L = Kg + size_t(p) * k * k;
    double* X = Li + size_t(p) * k * k;
    double* xc = trinv_col + size_t(w) * k;
    for (int i = lane; i < j; i += 32) X[size_t(i) * k + j] = 0.0;
    if (lane == 0) xc[j] = 1.0 / L[size_t(j) * k + j];
    __syncwarp();
    for (int i = j + 1; i < k; ++i) {
        const double* Li_row = L + size_t(i) * k;
        double part = 0.0;
        for (int a = j + lane; a < i; a += 32) part = fma(Li_row[a], xc[a], part);
        part = warp_sum_d(part);
        if (lane == 0) xc[i] = -part / Li_row[i];
        __syncwarp();
    }
    for (int i = j + lane; i < k; i += 32) X[size_t(i) * k + j] = xc[i];
}

// ---------------------------------------------------------------------------------------------
// 4. Jacobi diagonalisation of the symmetric kk x kk Rayleigh quotient (kk even; an odd k is
//    padded with an isolated zero row and column), one CTA per problem
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void rr_pair(int r, int t, int kk, int& p, int& q) {
    // circle method: index 0 stays, the others rotate one place per round
    const int n1 = kk - 1;
    if (t == 0) {
        p = 0;
        q = r % n1 + 1;
    } else {
        p = (t + r) % n1 + 1;
        q = (n1 - t + r) % n1 + 1;
    }
}

__global__ void __launch_bounds__(1024) fit_jacobi_kernel(double* Hm, double* Vm, double* ev, int k, int kk,
                                                           int col_warps) {
    extern __shared__ double rowbuf[];  // [col_warps][kk]
    double* H = Hm + size_t(blockIdx.x) * kk * kk;
    double* V = Vm + size_t(blockIdx.x) * kk * kk;
    // the round's active rotations (pairs with a rotation to apply), compacted
    __shared__ double act_c[kMaxK / 2], act_s[kMaxK / 2];
    __shared__ int act_p[kMaxK / 2], act_q[kMaxK / 2];
    __shared__ double red[32];
    __shared__ int nact, any_rot;
    const int tid = threadIdx.x, nt = blockDim.x, warp = tid >> 5, lane = tid & 31, nw = nt >> 5;
    // symmetrise the k x k block, zero the padding, V = I
    for (int e = tid; e < kk * kk; e += nt) {
        const int i = e / kk, j = e - i * kk;
        V[e] = i == j ? 1.0 : 0.0;
        if (i >= k || j >= k) {
            H[e] = 0.0;
        } else if (j < i) {
            const double v = 0.5 * (H[e] + H[size_t(j) * kk + i]);
            H[e] = v;
            H[size_t(j) * kk + i] = v;
        }
    }
    __syncthreads();
    const int half = kk / 2;
    for (int sweep = 0; sweep < kJacobiSweeps; ++sweep) {
        double off = 0.0, all = 0.0;
        for (int i = warp; i < kk; i += nw)
            for (int j = lane; j < kk; j += 32) {
                const double v = H[size_t(i) * kk + j];
                all += v * v;
                if (i != j) off += v * v;
            }
        off = block_sum(off, red);
        all = block_sum(all, red);
        if (off <= 1e-28 * all) break;  // off-diagonal norm <= 1e-14 of the whole
        // an entry below 1e-15 of the norm is rounding noise: rotating it away only moves the
        // noise elsewhere (entries of the smallest eigenvalues would otherwise never settle)
        const double floor_abs = 1e-15 * sqrt(all);
        if (tid == 0) any_rot = 0;
        for (int r = 0; r < kk - 1; ++r) {
            if (tid == 0) nact = 0;
            __syncthreads();
            for (int t = tid; t < half; t += nt) {  // the round's rotations (symmetric 2x2 Schur)
                int p, q;
                rr_pair(r, t, kk, p, q);
                const double apq = H[size_t(p) * kk + q], app = H[size_t(p) * kk + p], aqq = H[size_t(q) * kk + q];
                if (apq != 0.0 && fabs(apq) > fmax(1e-16 * sqrt(fabs(app * aqq)), floor_abs)) {
                    const double tau = (aqq - app) / (2.0 * apq);
                    const double tt = fabs(tau) > 1e150 ? 0.5 / tau
                                                        : (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
                    const double c = 1.0 / sqrt(1.0 + tt * tt);
                    const int a = atomicAdd(&nact, 1);
                    act_p[a] = p;
                    act_q[a] = q;
                    act_c[a] = c;
                    act_s[a] = tt * c;
                    any_rot = 1;
                }
            }
            __syncthreads();
            const int na = nact;
            if (na == 0) continue;  // uniform: every thread read nact after the barrier
            for (int a = warp; a < na; a += nw) {  // rows p, q: H <- Jᵀ H (contiguous rows)
                const int p = act_p[a], q = act_q[a];
                const double c = act_c[a], sn = act_s[a];
                double* hp = H + size_t(p) * kk;
                double* hq = H + size_t(q) * kk;
                for (int j0 = lane; j0 < kk; j0 += 32 * 8) {
                    double x[8], y[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int j = j0 + 32 * u;
                        x[u] = j < kk ? hp[j] : 0.0;
                        y[u] = j < kk ? hq[j] : 0.0;
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int j = j0 + 32 * u;
                        if (j < kk) {
                            hp[j] = c * x[u] - sn * y[u];
                            hq[j] = sn * x[u] + c * y[u];
                        }
                    }
                }
            }
            __syncthreads();
            // columns p, q of every row: H <- H J, V <- V J, two rows at a time per warp through
            // its shared-memory row buffers (contiguous loads and stores, both rows in flight)
            if (warp < col_warps) {
                double* rb0 = rowbuf + size_t(2 * warp) * kk;
                double* rb1 = rb0 + kk;
                for (int i = warp; i < 2 * kk; i += 2 * col_warps) {
                    const int i1 = i + col_warps;
                    const bool two = i1 < 2 * kk;
                    double* row0 = i < kk ? H + size_t(i) * kk : V + size_t(i - kk) * kk;
                    double* row1 = !two ? row0 : (i1 < kk ? H + size_t(i1) * kk : V + size_t(i1 - kk) * kk);
                    for (int j = lane; j < kk; j += 32) {
                        rb0[j] = row0[j];
                        if (two) rb1[j] = row1[j];
                    }
                    __syncwarp();
                    for (int a = lane; a < na; a += 32) {
                        const int p = act_p[a], q = act_q[a];
                        const double c = act_c[a], sn = act_s[a];
                        const double x0 = rb0[p], y0 = rb0[q];
                        rb0[p] = c * x0 - sn * y0;
                        rb0[q] = sn * x0 + c * y0;
                        if (two) {
                            const double x1 = rb1[p], y1 = rb1[q];
                            rb1[p] = c * x1 - sn * y1;
                            rb1[q] = sn * x1 + c * y1;
                        }
                    }
                    __syncwarp();
                    for (int j = lane; j < kk; j += 32) {
                        row0[j] = rb0[j];
                        if (two) row1[j] = rb1[j];
                    }
                    __syncwarp();
                }
            }
            __syncthreads();
        }
        if (!any_rot) break;
    }
    for (int c = tid; c < k; c += nt) ev[size_t(blockIdx.x) * kk + c] = H[size_t(c) * kk + c];
}

// top r Ritz pairs: rank by value (descending, ties by index); Vs = V[:, order] (k x r)
__global__ void __launch_bounds__(1024) fit_select_kernel(const double* ev, const double* Vm, int k, int kk, int r,
                                                          double* Vs, double* sig) {
    const int p = blockIdx.x;
    const double* e = ev + size_t(p) * kk;
    __shared__ int order[kMaxK];
    for (int c = threadIdx.x; c < k; c += blockDim.x) {
        const double v = e[c];
        int rank = 0;
        for (int c2 = 0; c2 < k; ++c2) {
            const double w = e[c2];
            rank += (w > v || (w == v && c2 < c)) ? 1 : 0;
        }
        if (rank < r) order[rank] = c;
    }
    __syncthreads();
    const double* V = Vm + size_t(p) * kk * kk;
    for (int idx = threadIdx.x; idx < k * r; idx += blockDim.x) {
        const int a = idx / r, c = idx - a * r;
        Vs[size_t(p) * k * r + idx] = V[size_t(a) * kk + order[c]];
    }
    for (int c = threadIdx.x; c < r; c += blockDim.x) sig[size_t(p) * r + c] = sqrt(fmax(e[order[c]], 0.0));
}

// 5. normalise each column of W (S x r), flip it so its largest-magnitude entry (first on ties)
//    is positive, write float W_down [S][r] and the singular values
__global__ void __launch_bounds__(256) fit_finalize_kernel(const double* Wd, const double* sig, int S, int r,
                                                           float* w_out, float* sig_out) {
    const int c = blockIdx.x, p = blockIdx.y;
    const double* W = Wd + size_t(p) * S * r;
    __shared__ double red[32];
    __shared__ double best_v[256];
    __shared__ int best_i[256];
    double ss = 0.0, bv = -1.0;
    int bi = 0x7fffffff;
    for (int i = threadIdx.x; i < S; i += 256) {
        const double v = W[size_t(i) * r + c];
        ss += v * v;
        if (fabs(v) > bv) {  // strictly larger keeps the first index within a thread
            bv = fabs(v);
            bi = i;
        }
    }
    const double nrm2 = block_sum(ss, red);
    best_v[threadIdx.x] = bv;
    best_i[threadIdx.x] = bi;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (threadIdx.x < o) {
            const double v2 = best_v[threadIdx.x + o];
            const int i2 = best_i[threadIdx.x + o];
            if (v2 > best_v[threadIdx.x] || (v2 == best_v[threadIdx.x] && i2 < best_i[threadIdx.x])) {
                best_v[threadIdx.x] = v2;
                best_i[threadIdx.x] = i2;
            }
        }
        __syncthreads();
    }
    const double nrm = sqrt(nrm2);
    const double sgn = W[size_t(best_i[0]) * r + c] < 0.0 ? -1.0 : 1.0;
    const double scale = nrm > 0.0 ? sgn / nrm : 0.0;
    for (int i = threadIdx.x; i < S; i += 256) w_out[(size_t(p) * S + i) * r + c] = float(W[size_t(i) * r + c] * scale);
    if (threadIdx.x == 0 && sig_out) sig_out[size_t(p) * r + c] = float(sig[size_t(p) * r + c]);
}

// ---------------------------------------------------------------------------------------------
// host driver
// ---------------------------------------------------------------------------------------------
struct FitDims {
    int m, k, kk;
    bool col;
};
FitDims fit_dims(int n, int S, int r) {
    FitDims d;
    d.m = n < S ? n : S;
    d.col = d.m == S;
    int k = 2 * r > r + kOver ? 2 * r : r + kOver;
    d.k = k < d.m ? k : d.m;
    d.kk = d.k + (d.k & 1);
    return d;
}

struct FitLayout {
    size_t mu, G, Z, Y, Kg, Li, H, V, ev, Vs, Wz, Wd, sig, total;
};
FitLayout fit_layout(int P, int n, int S, int r) {
    const FitDims d = fit_dims(n, S, r);
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t Pz = size_t(P), m = d.m, k = d.k, kk = d.kk;
    FitLayout L;
    size_t o = al(sizeof(lla_ws_header));
    auto take = [&](size_t doubles) {
        const size_t at = o;
        o = al(o + doubles * Pz * sizeof(double));
        return at;
    };
    L.mu = take(size_t(S));
    L.G = take(m * m);
    L.Z = take(m * k);
    L.Y = take(m * k);
    L.Kg = take(k * k);
    L.Li = take(k * k);
    L.H = take(kk * kk);
    L.V = take(kk * kk);
    L.ev = take(kk);
    L.Vs = take(k * size_t(r));
    L.Wz = take(m * size_t(r));
    L.Wd = take(size_t(S) * r);
    L.sig = take(size_t(r));
    L.total = o;
    return L;
}

template <class OA>
cudaError_t gemm(int P, int M, int N, int K, OA A, DOp B, double* C, long long c_batch, int ldc, cudaStream_t st) {
    dim3 grid((N + 63) / 64, (M + 63) / 64, P);
    fit_gemm_kernel<OA><<<grid, 64, 0, st>>>(M, N, K, A, B, C, c_batch, ldc);
    return cudaGetLastError();
}

}  // namespace

size_t lla_fit_workspace_bytes_impl(int P, int n, int S, int r) { return fit_layout(P, n, S, r).total; }

bool lla_fit_shape_ok(int n, int S, int r) {
    const FitDims d = fit_dims(n, S, r);
    return r <= d.m && d.k <= kMaxK;
}

lla_status lla_fit(int P, int n, int S, int r, const float* X, float* mu_out, float* w_out, float* sig_out, int iters,
                   void* workspace, cudaStream_t st) {
    const FitDims d = fit_dims(n, S, r);
    const FitLayout L = fit_layout(P, n, S, r);
    char* ws = static_cast<char*>(workspace);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws);
    auto buf = [&](size_t off) { return reinterpret_cast<double*>(ws + off); };
    double *mu = buf(L.mu), *G = buf(L.G), *Z = buf(L.Z), *Y = buf(L.Y), *Kg = buf(L.Kg), *Li = buf(L.Li);
    double *H = buf(L.H), *V = buf(L.V), *ev = buf(L.ev), *Vs = buf(L.Vs), *Wz = buf(L.Wz), *Wd = buf(L.Wd);
    double* sig = buf(L.sig);
    const int m = d.m, k = d.k, kk = d.kk;
    const long long mk = (long long)m * k, kk2 = (long long)k * k;
    LLA_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(lla_ws_header), st));
    // shared memory: the triangular inverse keeps one column per warp, the Jacobi column phase one
    // row per warp (at most ~200 KB)
    const int tri_warps = (200 * 1024) / (8 * k) < 32 ? (200 * 1024) / (8 * k) : 32;
    const size_t tri_smem = size_t(tri_warps) * k * sizeof(double);
    const int col_warps = (200 * 1024) / (16 * kk) < 32 ? (200 * 1024) / (16 * kk) : 32;
    const size_t jac_smem = size_t(2 * col_warps) * kk * sizeof(double);
    LLA_CUDA_TRY(cudaFuncSetAttribute(fit_trinv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(tri_smem)));
    LLA_CUDA_TRY(cudaFuncSetAttribute(fit_jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(jac_smem)));

    fit_mean_kernel<<<dim3((S + 255) / 256, P), 256, 0, st>>>(X, n, S, mu, mu_out);
    LLA_CUDA_TRY(cudaGetLastError());
    const int tiles = (m + 63) / 64;
    fit_gram_kernel<<<dim3(tiles * (tiles + 1) / 2, P), 256, 0, st>>>(X, mu, n, S, m, d.col ? 1 : 0, G);
    LLA_CUDA_TRY(cudaGetLastError());
    fit_init_kernel<<<dim3(unsigned((mk + 255) / 256), P), 256, 0, st>>>(Y, m, k);
    LLA_CUDA_TRY(cudaGetLastError());

    // one Cholesky QR pass: dst = src L⁻ᵀ with L Lᵀ = srcᵀ src (+ shift)
    auto cholqr = [&](const double* src, double* dst, bool shifted) -> lla_status {
        LLA_CUDA_TRY(gemm(P, k, k, m, DOp{src, mk, 1, k}, DOp{src, mk, k, 1}, Kg, kk2, k, st));
        fit_chol_kernel<<<P, 1024, 0, st>>>(Kg, k, m, shifted ? 1 : 0, status);
        LLA_CUDA_TRY(cudaGetLastError());
        fit_trinv_kernel<<<dim3((k + tri_warps - 1) / tri_warps, P), 32 * tri_warps, tri_smem, st>>>(Kg, Li, k);
        LLA_CUDA_TRY(cudaGetLastError());
        LLA_CUDA_TRY(gemm(P, m, k, k, DOp{src, mk, k, 1}, DOp{Li, kk2, 1, k}, dst, mk, k, st));
        return LLA_OK;
    };
    // shifted CholeskyQR3 of Y into Z (Y is overwritten)
    auto orth = [&]() -> lla_status {
        lla_status s;
        if ((s = cholqr(Y, Z, true)) != LLA_OK) return s;
        if ((s = cholqr(Z, Y, false)) != LLA_OK) return s;
        return cholqr(Y, Z, false);
    };
    lla_status s;
    if ((s = orth()) != LLA_OK) return s;
    // `iters` products with G; an orthonormalisation after every second one (G² Z spans the same
    // block as G (G Z) orthonormalised, and shifted CholeskyQR3 takes the squared conditioning)
    for (int it = 0; it < iters; it += 2) {
        if (it + 1 < iters) {
            LLA_CUDA_TRY(gemm(P, m, k, m, DOp{G, (long long)m * m, m, 1}, DOp{Z, mk, k, 1}, Y, mk, k, st));
            LLA_CUDA_TRY(gemm(P, m, k, m, DOp{G, (long long)m * m, m, 1}, DOp{Y, mk, k, 1}, Z, mk, k, st));
            LLA_CUDA_TRY(cudaMemcpyAsync(Y, Z, size_t(P) * mk * sizeof(double), cudaMemcpyDeviceToDevice, st));
        } else {
            LLA_CUDA_TRY(gemm(P, m, k, m, DOp{G, (long long)m * m, m, 1}, DOp{Z, mk, k, 1}, Y, mk, k, st));
        }
        if ((s = orth()) != LLA_OK) return s;
    }
    // Rayleigh–Ritz
    LLA_CUDA_TRY(gemm(P, m, k, m, DOp{G, (long long)m * m, m, 1}, DOp{Z, mk, k, 1}, Y, mk, k, st));
    LLA_CUDA_TRY(gemm(P, k, k, m, DOp{Z, mk, 1, k}, DOp{Y, mk, k, 1}, H, (long long)kk * kk, kk, st));
    fit_jacobi_kernel<<<P, 1024, jac_smem, st>>>(H, V, ev, k, kk, col_warps);
    LLA_CUDA_TRY(cudaGetLastError());
    fit_select_kernel<<<P, 1024, 0, st>>>(ev, V, k, kk, r, Vs, sig);
    LLA_CUDA_TRY(cudaGetLastError());
    LLA_CUDA_TRY(gemm(P, m, r, k, DOp{Z, mk, k, 1}, DOp{Vs, (long long)k * r, r, 1}, Wz, (long long)m * r, r, st));
    const double* W = Wz;
    if (!d.col) {  // left singular vectors of Xc: W = Xcᵀ U, normalised below
        LLA_CUDA_TRY(gemm(P, S, r, n, XcT{X, mu, n, S}, DOp{Wz, (long long)m * r, r, 1}, Wd, (long long)S * r, r, st));
        W = Wd;
    }
    fit_finalize_kernel<<<dim3(r, P), 256, 0, st>>>(W, sig, S, r, w_out, sig_out);
    LLA_CUDA_TRY(cudaGetLastError());
    return LLA_OK;
}
