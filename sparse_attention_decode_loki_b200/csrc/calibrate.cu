// Offline PCA calibration of Loki: per KV head, the principal components of
// calibration keys (NeurIPS 2024 poster page, "Visual Insights" Figure 1
// caption: offline PCA on keys gathered from a calibration set; study.space
// summary: PCA reduces the key dimensionality).
//
// 1. k_mean:  mu = mean of the N keys (fp64).
// 2. k_cov:   C = (X - mu)^T (X - mu) / (N - 1), 16x16 output tiles, fp64.
// 3. k_jacobi: cyclic Jacobi eigen-decomposition of C in fp64 (Golub & Van
//    Loan, "Matrix Computations", symmetric Schur 2x2 rotation and the
//    parallel round-robin ordering): each round pairs all D indices into D/2
//    disjoint (p, q) pairs, zeroes every A[p][q] at once with a column pass
//    then a row pass, and accumulates the rotations into V. Sweeps stop when
//    the off-diagonal Frobenius norm is below 1e-14 of the total, or after
//    kMaxSweeps. A lives in shared memory; V (transposed, fp64) in the
//    workspace. Finally eigenvalues are ranked descending, each vector is
//    signed so its largest-magnitude entry (lowest index on a tie) is
//    positive, and P = [v_0 ... v_{D-1}] is written as fp32.
// Offline and off the decode path: written for clarity, not speed.
#include "common.cuh"
#include "launch.h"

namespace loki {

constexpr int kMaxSweeps = 40;

template <class E>
__global__ void k_mean(const typename E::T* __restrict__ X, int64_t N, int H, int D,
                       double* __restrict__ mu) {
    const int h = blockIdx.x, c = threadIdx.x;
    if (c >= D) return;
    double s = 0.0;
    for (int64_t n = 0; n < N; ++n) s += (double)E::load1(X + (n * H + h) * D + c);
    mu[(int64_t)h * D + c] = s / (double)N;
}

template <class E>
__global__ void __launch_bounds__(256) k_cov(const typename E::T* __restrict__ X, int64_t N, int H,
                                             int D, const double* __restrict__ mu,
                                             double* __restrict__ C) {
    __shared__ double xi[16][17], xj[16][17];
    const int h = blockIdx.z;
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int ib = blockIdx.y * 16, jb = blockIdx.x * 16;
    const double mui = mu[(int64_t)h * D + ib + tx];
    const double muj = mu[(int64_t)h * D + jb + tx];
    double acc = 0.0;
    for (int64_t n0 = 0; n0 < N; n0 += 16) {
        const int64_t n = n0 + ty;
        double a = 0.0, b = 0.0;
        if (n < N) {
            a = (double)E::load1(X + (n * H + h) * D + ib + tx) - mui;
            b = (double)E::load1(X + (n * H + h) * D + jb + tx) - muj;
        }
        xi[ty][tx] = a;
        xj[ty][tx] = b;
        __syncthreads();
#pragma unroll
        for (int nn = 0; nn < 16; ++nn) acc = fma(xi[nn][ty], xj[nn][tx], acc);
        __syncthreads();
    }
    C[((int64_t)h * D + ib + ty) * D + jb + tx] = acc / (double)(N - 1);
}

// position of slot m in round `round` of the circle-method round robin over
// D indices (slot 0 fixed, the other D - 1 rotate)
__device__ __forceinline__ int rr_pos(int m, int round, int D) {
    return m == 0 ? 0 : 1 + (m - 1 + round) % (D - 1);
}

__device__ double block_sum(double v, double* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = (blockDim.x + 31) >> 5;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = 0.0;
    for (int i = 0; i < nw; ++i) t += red[i];
    return t;
}

__global__ void __launch_bounds__(1024) k_jacobi(const double* __restrict__ Cg,
                                                 double* __restrict__ Vt_g, float* __restrict__ P,
                                                 float* __restrict__ eig, int D) {
    extern __shared__ double A[];  // D x (D + 1)
    __shared__ double s_c[64], s_s[64];
    __shared__ int s_p[64], s_q[64];
    __shared__ double red[32];
    const int h = blockIdx.x;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int ld = D + 1;
    const int half = D / 2;
    const double* C = Cg + (int64_t)h * D * D;
    double* Vt = Vt_g + (int64_t)h * D * D;  // Vt[c][i] = V[i][c]

    for (int it = tid; it < D * D; it += nt) {
        const int i = it / D, j = it % D;
        A[i * ld + j] = C[it];
        Vt[it] = (i == j) ? 1.0 : 0.0;
    }
    __syncthreads();

    for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
        double off = 0.0, tot = 0.0;
        for (int it = tid; it < D * D; it += nt) {
            const int i = it / D, j = it % D;
            const double a = A[i * ld + j];
            tot += a * a;
            if (i != j) off += a * a;
        }
        off = block_sum(off, red);
        tot = block_sum(tot, red);
        if (off <= 1e-28 * tot) break;

        for (int round = 0; round < D - 1; ++round) {
            if (tid < half) {
                int p = rr_pos(tid, round, D), q = rr_pos(D - 1 - tid, round, D);
                if (p > q) {
                    const int x = p;
                    p = q;
                    q = x;
                }
                const double app = A[p * ld + p], aqq = A[q * ld + q], apq = A[p * ld + q];
                double c = 1.0, s = 0.0;
                if (apq != 0.0) {
                    const double tau = (aqq - app) / (2.0 * apq);
                    const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + hypot(1.0, tau));
                    c = 1.0 / sqrt(1.0 + t * t);
                    s = t * c;
                }
                s_p[tid] = p;
                s_q[tid] = q;
                s_c[tid] = c;
                s_s[tid] = s;
            }
            __syncthreads();
            // columns p, q of A and of V:  [a_p a_q] <- [a_p a_q] [[c, s], [-s, c]]
            for (int it = tid; it < half * D; it += nt) {
                const int k = it / D, row = it % D;
                const int p = s_p[k], q = s_q[k];
                const double c = s_c[k], s = s_s[k];
                const double a = A[row * ld + p], b = A[row * ld + q];
                A[row * ld + p] = c * a - s * b;
                A[row * ld + q] = s * a + c * b;
                const double va = Vt[(int64_t)p * D + row], vb = Vt[(int64_t)q * D + row];
                Vt[(int64_t)p * D + row] = c * va - s * vb;
                Vt[(int64_t)q * D + row] = s * va + c * vb;
            }
            __syncthreads();
            // rows p, q of A:  [a_p; a_q] <- [[c, -s], [s, c]] [a_p; a_q]
            for (int it = tid; it < half * D; it += nt) {
                const int k = it / D, col = it % D;
                const int p = s_p[k], q = s_q[k];
                const double c = s_c[k], s = s_s[k];
                const double a = A[p * ld + col], b = A[q * ld + col];
                A[p * ld + col] = c * a - s * b;
                A[q * ld + col] = s * a + c * b;
            }
            __syncthreads();
        }
    }

    if (tid < D) {
        const double w = A[tid * ld + tid];
        int rank = 0;
        for (int j = 0; j < D; ++j) {
            const double x = A[j * ld + j];
            rank += (x > w) || (x == w && j < tid);
        }
        const double* v = Vt + (int64_t)tid * D;
        int imax = 0;
        double vmax = fabs(v[0]);
        for (int i = 1; i < D; ++i) {
            if (fabs(v[i]) > vmax) {
                vmax = fabs(v[i]);
                imax = i;
            }
        }
        const double sgn = v[imax] < 0.0 ? -1.0 : 1.0;
        float* Ph = P + (int64_t)h * D * D;
        for (int i = 0; i < D; ++i) Ph[(int64_t)i * D + rank] = (float)(sgn * v[i]);
        if (eig) eig[(int64_t)h * D + rank] = (float)w;
    }
}

cudaError_t launch_calibrate(Dt dt, const void* keys, int64_t N, int H_kv, int D, float* P,
                             float* eigvals, double* ws_mean, double* ws_cov, double* ws_vec,
                             cudaStream_t s) {
    if (dt == kF32)
        k_mean<ElemF32><<<H_kv, 128, 0, s>>>(static_cast<const float*>(keys), N, H_kv, D, ws_mean);
    else
        k_mean<ElemBF16><<<H_kv, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(keys), N, H_kv, D,
                                              ws_mean);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 cgrid(D / 16, D / 16, H_kv), cblock(16, 16);
    if (dt == kF32)
        k_cov<ElemF32><<<cgrid, cblock, 0, s>>>(static_cast<const float*>(keys), N, H_kv, D,
                                                ws_mean, ws_cov);
    else
        k_cov<ElemBF16><<<cgrid, cblock, 0, s>>>(static_cast<const __nv_bfloat16*>(keys), N, H_kv,
                                                 D, ws_mean, ws_cov);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = (size_t)D * (D + 1) * sizeof(double);
    e = cudaFuncSetAttribute(k_jacobi, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_jacobi<<<H_kv, 1024, smem, s>>>(ws_cov, ws_vec, P, eigvals, D);
    return cudaGetLastError();
}

}  // namespace loki
