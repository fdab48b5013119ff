// Device compressor, first step: the top-r singular triplets of a tenant's delta on the GPU.
//
// "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法", section "Delta-CoMe的技术原理", and
// "Delta-CoMe: Training-Free Delta-Compression with Mixed-Precision for Large Language Models",
// section "Approach": the delta W_ft - W_base is decomposed by SVD before its singular vectors are
// quantised.  Only the top r = (ranks the bit plan keeps) triplets are needed, so the device path
// is a randomized range finder with power iterations (Halko, Martinsson and Tropp, "Finding
// structure with randomness", SIAM Review 53(2), 2011, algorithms 4.4 and 5.1):
//   Delta = W_ft - W_base;  Y = Delta Omega (Omega Gaussian, d_in x l, l = r + oversampling);
//   Q = orth(Y);  q times: Q' = orth(Delta^T Q), Q = orth(Delta Q');
//   B^T = Delta^T Q;  SVD of B by one-sided Jacobi (Hestenes): B^T J = W with orthogonal columns,
//   sigma_j = |W_j|, v_j = W_j / sigma_j, u_j = Q J_j;  the r largest, signs fixed as the oracle
//   does (the largest-magnitude entry of v_i positive, the lowest index on ties).
// orth() is CholeskyQR2: the Gram matrix in fp64, its Cholesky factor, the basis multiplied by the
// factor's inverse, twice (bases of more than 4096 columns fall back to one-sided Jacobi).  Matrices
// whose columns the algorithm works on are stored transposed, one column per contiguous row, so
// every Jacobi pair reads two contiguous rows.  Products run on an fp32 tiled GEMM; Gram matrices,
// Cholesky and Jacobi sums are fp64.  The library allocates nothing: the caller passes a workspace
// of dc_svd_workspace_size bytes.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "dc.h"
#include "dc_internal.h"

namespace {

constexpr int kTile = 64, kTK = 16;

// C[M x N] = A[M x K] * B[K x N] (TRANS_B false, B row-major K x N) or A * B^T (TRANS_B true,
// B row-major N x K).  Row-major everything, fp32, 64 x 64 tiles, 4 x 4 outputs per thread.
template <bool TRANS_B>
__global__ void __launch_bounds__(256) k_sgemm(const float* __restrict__ A, const float* __restrict__ B,
                                               float* __restrict__ Cm, int M, int N, int K, int lda, int ldb,
                                               int ldc) {
  __shared__ float As[kTK][kTile + 4];
  __shared__ float Bs[kTK][kTile + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * kTile, n0 = blockIdx.x * kTile;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kTK) {
    for (int i = tid; i < kTile * kTK; i += 256) {  // A tile: 64 rows x 16 k
      const int r = i / kTK, k = i % kTK;
      const int gm = m0 + r, gk = k0 + k;
      As[k][r] = (gm < M && gk < K) ? A[(int64_t)gm * lda + gk] : 0.f;
    }
    for (int i = tid; i < kTile * kTK; i += 256) {
      int k, c;
      if (TRANS_B) {
        c = i / kTK, k = i % kTK;  // B[n][k], k contiguous
      } else {
        k = i / kTile, c = i % kTile;  // B[k][n], n contiguous
      }
      const int gn = n0 + c, gk = k0 + k;
      float v = 0.f;
      if (gn < N && gk < K) v = TRANS_B ? B[(int64_t)gn * ldb + gk] : B[(int64_t)gk * ldb + gn];
      Bs[k][c] = v;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kTK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty + 16 * i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx + 16 * j;
      if (gn < N) Cm[(int64_t)gm * ldc + gn] = acc[i][j];
    }
  }
}

// Delta = W_ft - W_base, fp32 row-major [d_out, d_in].
__global__ void k_svd_delta(const void* __restrict__ wft, const void* __restrict__ wb, int dtype, float* __restrict__ D,
                            int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    float a, b;
    if (dtype == DC_DTYPE_BF16) {
      a = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(wft)[i]);
      b = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(wb)[i]);
    } else {
      a = reinterpret_cast<const float*>(wft)[i];
      b = reinterpret_cast<const float*>(wb)[i];
    }
    D[i] = a - b;
  }
}

// Omega^T [l x d_in]: standard normal values from a counter-based generator (SplitMix64 of
// seed + index, two 32-bit halves to Box-Muller).  SplitMix64: Steele, Lea and Flood, "Fast
// splittable pseudorandom number generators", OOPSLA 2014.
__device__ __forceinline__ uint64_t svd_mix64(uint64_t z) {
  z += 0x9e3779b97f4a7c15ull;
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
  return z ^ (z >> 31);
}
__global__ void k_svd_gauss(float* __restrict__ out, int64_t n, uint64_t seed) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t z = svd_mix64(seed * 0x632be59bd9b4e019ull + (uint64_t)i);
    const float u1 = ((float)(uint32_t)(z >> 40) + 1.f) * (1.f / 16777217.f);  // (0, 1]
    const float u2 = (float)(uint32_t)(z & 0xffffffu) * (1.f / 16777216.f);
    out[i] = sqrtf(-2.f * logf(u1)) * cospif(2.f * u2);
  }
}

__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  double s = 0.0;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += red[i];
  return s;
}

// One round of the cyclic one-sided Jacobi sweep over the n rows of M (each row one column of the
// matrix being orthogonalised, length m): block i takes pair i of round `round` of the round-robin
// tournament over npad = n rounded up to even (slot npad - 1 fixed, the others rotating); pairs
// holding the pad slot are skipped.  A pair whose normalised inner product |g| / sqrt(a b) exceeds
// tol is rotated, and the same rotation is applied to rows of Jt (n x n) if given.  The largest
// normalised inner product of the round goes to *offmax (as float bits; values are >= 0).
__global__ void __launch_bounds__(256) k_jacobi_round(float* __restrict__ M, int n, int m, float* __restrict__ Jt,
                                                      int round, float tol, int* __restrict__ offmax) {
  __shared__ double red[8];
  const int npad = n + (n & 1);
  const int i = blockIdx.x;
  int a, b;
  if (i == 0) {
    a = round;
    b = npad - 1;
  } else {
    a = (round + i) % (npad - 1);
    b = (round - i + npad - 1) % (npad - 1);
  }
  if (a >= n || b >= n) return;
  float* Ma = M + (int64_t)a * m;
  float* Mb = M + (int64_t)b * m;
  double al = 0.0, be = 0.0, ga = 0.0;
  for (int k = threadIdx.x; k < m; k += blockDim.x) {
    const double x = Ma[k], y = Mb[k];
    al += x * x;
    be += y * y;
    ga += x * y;
  }
  al = block_sum(al, red);
  be = block_sum(be, red);
  ga = block_sum(ga, red);
  const double den = sqrt(al * be);
  const double rel = den > 0.0 ? fabs(ga) / den : 0.0;
  if (threadIdx.x == 0) atomicMax(offmax, __float_as_int((float)rel));
  if (!(rel > tol)) return;
  const double zeta = (be - al) / (2.0 * ga);
  const double t = (zeta >= 0.0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
  const float c = (float)(1.0 / sqrt(1.0 + t * t)), s = (float)(t / sqrt(1.0 + t * t));
  for (int k = threadIdx.x; k < m; k += blockDim.x) {
    const float x = Ma[k], y = Mb[k];
    Ma[k] = c * x - s * y;
    Mb[k] = s * x + c * y;
  }
  if (Jt) {
    float* Ja = Jt + (int64_t)a * n;
    float* Jb = Jt + (int64_t)b * n;
    for (int k = threadIdx.x; k < n; k += blockDim.x) {
      const float x = Ja[k], y = Jb[k];
      Ja[k] = c * x - s * y;
      Jb[k] = s * x + c * y;
    }
  }
}

// Row norms of M [n x m] into nrm (fp64 sums); with `normalize`, rows are scaled to unit length
// (rows of zero norm stay zero).
__global__ void __launch_bounds__(256) k_row_norms(float* __restrict__ M, int m, float* __restrict__ nrm, int normalize) {
  __shared__ double red[8];
  float* R = M + (int64_t)blockIdx.x * m;
  double s = 0.0;
  for (int k = threadIdx.x; k < m; k += blockDim.x) s += (double)R[k] * R[k];
  s = block_sum(s, red);
  const float v = (float)sqrt(s);
  if (threadIdx.x == 0) nrm[blockIdx.x] = v;
  if (normalize && v > 0.f) {
    const float inv = 1.f / v;
    for (int k = threadIdx.x; k < m; k += blockDim.x) R[k] *= inv;
  }
}

// ---- CholeskyQR2 for the range finder's bases (orthonormal rows of M, n x m):
//   G = M M^T (fp64), G = L L^T, M <- L^-1 M, twice (the second pass repairs the first's
//   rounding; Fukaya, Nakatsukasa, Yanagisawa, Yamamoto, "CholeskyQR2", ScalA 2014).
// Its cost is two Gram products and two small triangular steps, against O(n^2 m) per sweep for
// the one-sided Jacobi, which remains the method for the final SVD of B.

// G = M M^T in fp64 (M rows of length m, fp32): 32 x 32 output tiles, upper tiles only, mirrored.
__global__ void __launch_bounds__(256) k_gram64(const float* __restrict__ M, int n, int m, double* __restrict__ G) {
  const int bi = blockIdx.y, bj = blockIdx.x;
  if (bj < bi) return;
  __shared__ float A[32][33], B[32][33];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double acc[2][2] = {};
  for (int k0 = 0; k0 < m; k0 += 32) {
    for (int e = threadIdx.x; e < 32 * 32; e += 256) {
      const int r = e >> 5, c = e & 31;
      const int ra = 32 * bi + r, rb = 32 * bj + r, k = k0 + c;
      A[r][c] = (ra < n && k < m) ? M[(int64_t)ra * m + k] : 0.f;
      B[r][c] = (rb < n && k < m) ? M[(int64_t)rb * m + k] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      const double a0 = A[ty][k], a1 = A[ty + 16][k], b0 = B[tx][k], b1 = B[tx + 16][k];
      acc[0][0] = fma(a0, b0, acc[0][0]);
      acc[0][1] = fma(a0, b1, acc[0][1]);
      acc[1][0] = fma(a1, b0, acc[1][0]);
      acc[1][1] = fma(a1, b1, acc[1][1]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int i = 32 * bi + ty + 16 * a, j = 32 * bj + tx + 16 * b;
      if (i < n && j < n) {
        G[(int64_t)i * n + j] = acc[a][b];
        G[(int64_t)j * n + i] = acc[a][b];
      }
    }
}

// Diagonal shift of G by eps * trace / n (keeps the factorisation defined when M's rows are nearly
// dependent; those directions then get no weight in the range).  One block.
__global__ void k_gram_shift(double* __restrict__ G, int n, double eps) {
  __shared__ double red[8];
  double t = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) t += G[(int64_t)i * n + i];
  t = block_sum(t, red);
  const double sh = eps * (t > 0.0 ? t / n : 1.0);
  for (int i = threadIdx.x; i < n; i += blockDim.x) G[(int64_t)i * n + i] += sh;
}

// Step k of the right-looking Cholesky on the lower triangle: G[i][j] -= G[i][k] G[j][k] / G[k][k]
// for k < j <= i (column k itself stays as it is; the factor is read off at the end).
__global__ void k_chol_step(double* __restrict__ G, int n, int k) {
  const int64_t w = n - k - 1;
  const int64_t tot = w * (w + 1) / 2;
  const double inv = 1.0 / G[(int64_t)k * n + k];
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < tot; e += (int64_t)gridDim.x * blockDim.x) {
    // e -> (a, b), 0 <= b <= a < w, row-major over the triangle
    int64_t a = (int64_t)((sqrt(8.0 * (double)e + 1.0) - 1.0) * 0.5);
    while (a * (a + 1) / 2 > e) --a;
    while ((a + 1) * (a + 2) / 2 <= e) ++a;
    const int64_t b = e - a * (a + 1) / 2;
    const int i = k + 1 + (int)a, j = k + 1 + (int)b;
    G[(int64_t)i * n + j] -= G[(int64_t)i * n + k] * G[(int64_t)j * n + k] * inv;
  }
}

// L[i][k] = G[i][k] / sqrt(G[k][k]) for i >= k (the Cholesky factor, in place, lower triangle);
// a non-positive pivot is reported in *bad.
__global__ void k_chol_finish(double* __restrict__ G, int n, int* __restrict__ bad) {
  const int64_t tot = (int64_t)n * n;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < tot; e += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / n), k = (int)(e % n);
    if (k > i) continue;
    const double d = G[(int64_t)k * n + k];
    if (!(d > 0.0)) {
      if (i == k) atomicExch(bad, 1);
      continue;
    }
    G[e] = G[e] / sqrt(d);  // the diagonal becomes sqrt(d) too
  }
}

// X = L^-1 (lower triangular, fp32 out): block j solves L x = e_j by forward substitution.
__global__ void __launch_bounds__(256) k_trinv(const double* __restrict__ L, int n, float* __restrict__ X) {
  __shared__ double red[8];
  __shared__ double xs[4096];
  const int j = blockIdx.x;
  for (int i = threadIdx.x; i < n; i += blockDim.x) X[(int64_t)i * n + j] = 0.f;
  if (threadIdx.x == 0) xs[j] = 1.0 / L[(int64_t)j * n + j];
  __syncthreads();
  for (int i = j + 1; i < n; ++i) {
    double sacc = 0.0;
    for (int t = j + threadIdx.x; t < i; t += blockDim.x) sacc += L[(int64_t)i * n + t] * xs[t];
    sacc = block_sum(sacc, red);
    if (threadIdx.x == 0) xs[i] = -sacc / L[(int64_t)i * n + i];
    __syncthreads();
  }
  for (int i = j + threadIdx.x; i < n; i += blockDim.x) X[(int64_t)i * n + j] = (float)xs[i];
}

__global__ void k_identity(float* __restrict__ J, int n) {
  const int64_t total = (int64_t)n * n;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x)
    J[i] = (i / n == i % n) ? 1.f : 0.f;
}

// Outputs: rank of every sigma (descending, lower index first on ties) -> the r largest triplets:
// S[i], Vt[i] = W_j / sigma_j, U[i] = Ut_j, then the sign rule (largest |v| entry positive, lowest
// index on ties).  One block per candidate j.
__global__ void __launch_bounds__(256) k_svd_emit(const float* __restrict__ sig, int l, int r,
                                                  const float* __restrict__ Wt, int d_in,
                                                  const float* __restrict__ Ut, int d_out, float* __restrict__ U,
                                                  float* __restrict__ S, float* __restrict__ Vt) {
  __shared__ int s_rank;
  __shared__ float s_val[8];
  __shared__ int s_idx[8];
  const int j = blockIdx.x;
  const float sj = sig[j];
  int cnt = 0;
  for (int k = threadIdx.x; k < l; k += blockDim.x) {
    const float sk = sig[k];
    cnt += (sk > sj || (sk == sj && k < j)) ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (threadIdx.x == 0) s_rank = 0;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) atomicAdd(&s_rank, cnt);
  __syncthreads();
  const int rank = s_rank;
  if (rank >= r) return;
  const float* w = Wt + (int64_t)j * d_in;
  const float inv = sj > 0.f ? 1.f / sj : 0.f;
  // largest |v| entry, lowest index on ties
  float best = -1.f;
  int bi = 0;
  for (int k = threadIdx.x; k < d_in; k += blockDim.x) {
    const float v = fabsf(w[k]);
    if (v > best) {
      best = v;
      bi = k;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > best || (ov == best && oi < bi)) {
      best = ov;
      bi = oi;
    }
  }
  if ((threadIdx.x & 31) == 0) {
    s_val[threadIdx.x >> 5] = best;
    s_idx[threadIdx.x >> 5] = bi;
  }
  __syncthreads();
  float bv = s_val[0];
  int bx = s_idx[0];
  for (int i = 1; i < (int)(blockDim.x >> 5); ++i)
    if (s_val[i] > bv || (s_val[i] == bv && s_idx[i] < bx)) {
      bv = s_val[i];
      bx = s_idx[i];
    }
  const float sg = w[bx] < 0.f ? -1.f : 1.f;
  if (threadIdx.x == 0) S[rank] = sj;
  for (int k = threadIdx.x; k < d_in; k += blockDim.x) Vt[(int64_t)rank * d_in + k] = sg * w[k] * inv;
  const float* u = Ut + (int64_t)j * d_out;
  for (int k = threadIdx.x; k < d_out; k += blockDim.x) U[(int64_t)rank * d_out + k] = sg * u[k];
}

struct SvdWs {
  int64_t delta, qt, zt, jt, ut, sig, gram, tinv, off, total;
};

SvdWs svd_ws(int d_out, int d_in, int l) {
  SvdWs W;
  int64_t o = 0;
  auto take = [&](int64_t bytes) {
    const int64_t r = o;
    o = (o + bytes + 255) / 256 * 256;
    return r;
  };
  W.delta = take((int64_t)d_out * d_in * 4);
  W.qt = take((int64_t)l * d_out * 4);
  W.zt = take((int64_t)l * d_in * 4);
  W.jt = take((int64_t)l * l * 4);
  W.ut = take((int64_t)l * std::max(d_out, d_in) * 4);  // U^T at the end; scratch of the range finder
  W.sig = take((int64_t)l * 4);
  W.gram = take((int64_t)l * l * 8);
  W.tinv = take((int64_t)l * l * 4);
  W.off = take(256);
  W.total = o;
  return W;
}

int svd_l(int d_out, int d_in, int r, int oversample) {
  return std::min(std::min(d_out, d_in), r + std::max(0, oversample));
}

template <bool TB>
dc_status gemm(const float* A, const float* B, float* C, int M, int N, int K, int lda, int ldb, int ldc,
               cudaStream_t s) {
  const dim3 grid((N + kTile - 1) / kTile, (M + kTile - 1) / kTile);
  k_sgemm<TB><<<grid, 256, 0, s>>>(A, B, C, M, N, K, lda, ldb, ldc);
  return dc_cuda_check(cudaGetLastError(), "svd gemm");
}

// One-sided Jacobi on the n rows (length m) of M until the largest normalised inner product of a
// sweep is at most tol (or max_sweeps).  Synchronises the stream once per sweep.
dc_status jacobi(float* M, int n, int m, float* Jt, float tol, int max_sweeps, int* off_dev, cudaStream_t s,
                 int* sweeps_out) {
  const int npad = n + (n & 1);
  int sweeps = 0;
  for (; sweeps < max_sweeps; ++sweeps) {
    dc_status st = dc_cuda_check(cudaMemsetAsync(off_dev, 0, 4, s), "jacobi reset");
    if (st) return st;
    for (int round = 0; round < npad - 1; ++round) k_jacobi_round<<<npad / 2, 256, 0, s>>>(M, n, m, Jt, round, tol, off_dev);
    st = dc_cuda_check(cudaGetLastError(), "jacobi round");
    if (st) return st;
    int offbits = 0;
    st = dc_cuda_check(cudaMemcpyAsync(&offbits, off_dev, 4, cudaMemcpyDeviceToHost, s), "jacobi read");
    if (st) return st;
    st = dc_cuda_check(cudaStreamSynchronize(s), "jacobi sync");
    if (st) return st;
    float off;
    std::memcpy(&off, &offbits, 4);
    if (!(off > tol)) {
      ++sweeps;
      break;
    }
  }
  if (sweeps_out) *sweeps_out += sweeps;
  return DC_OK;
}

// Orthonormal rows of M (n x m) spanning the same space, by CholeskyQR2; tmp: n x m fp32 scratch.
// Synchronises the stream (to read the pivot flag).
dc_status orth_cholqr2(float* M, int n, int m, float* tmp, double* G, float* X, int* bad, cudaStream_t s) {
  if (n > 4096) {  // beyond k_trinv's shared vector: one-sided Jacobi, then unit rows
    int sw = 0;
    dc_status st = jacobi(M, n, m, nullptr, 1e-6f, 40, bad, s, &sw);
    if (st) return st;
    k_row_norms<<<n, 256, 0, s>>>(M, m, reinterpret_cast<float*>(G), 1);
    return dc_cuda_check(cudaGetLastError(), "orth norms");
  }
  dc_status st = dc_cuda_check(cudaMemsetAsync(bad, 0, 4, s), "orth flag");
  if (st) return st;
  for (int pass = 0; pass < 2; ++pass) {
    const dim3 gg((n + 31) / 32, (n + 31) / 32);
    k_gram64<<<gg, 256, 0, s>>>(M, n, m, G);
    k_gram_shift<<<1, 256, 0, s>>>(G, n, 1e-13);
    for (int k = 0; k + 1 < n; ++k) {
      const int64_t w = n - k - 1, tot = w * (w + 1) / 2;
      k_chol_step<<<(unsigned)std::min<int64_t>((tot + 255) / 256, 148 * 8), 256, 0, s>>>(G, n, k);
    }
    k_chol_finish<<<(unsigned)std::min<int64_t>(((int64_t)n * n + 255) / 256, 148 * 8), 256, 0, s>>>(G, n, bad);
    k_trinv<<<n, 256, 0, s>>>(G, n, X);
    if ((st = gemm<false>(X, M, tmp, n, m, n, n, m, m, s))) return st;
    st = dc_cuda_check(cudaMemcpyAsync(M, tmp, (size_t)n * m * 4, cudaMemcpyDeviceToDevice, s), "orth copy");
    if (st) return st;
  }
  int hbad = 0;
  st = dc_cuda_check(cudaMemcpyAsync(&hbad, bad, 4, cudaMemcpyDeviceToHost, s), "orth flag read");
  if (st) return st;
  st = dc_cuda_check(cudaStreamSynchronize(s), "orth sync");
  if (st) return st;
  if (hbad) return dc_fail(DC_ERR_INVALID_ARG, "svd: the range basis lost rank (Cholesky pivot <= 0)");
  return DC_OK;
}

}  // namespace

extern "C" size_t dc_svd_workspace_size(int32_t d_out, int32_t d_in, int32_t r, int32_t oversample) {
  DC_NVTX("dc_svd_workspace_size");
  if (d_out <= 0 || d_in <= 0 || r <= 0 || r > std::min(d_out, d_in) || oversample < 0) return 0;
  return (size_t)svd_ws(d_out, d_in, svd_l(d_out, d_in, r, oversample)).total;
}

extern "C" dc_status dc_svd_device(const void* W_ft, const void* W_base, int32_t dtype, int32_t d_out, int32_t d_in,
                                   int32_t r, int32_t oversample, int32_t power_iters, uint64_t seed, float* U_out,
                                   float* S_out, float* Vt_out, void* ws, size_t ws_bytes, void* stream,
                                   int32_t* sweeps_out) {
  DC_NVTX("dc_svd_device");
  dc_clear_error();
  if (!W_ft || !W_base || !U_out || !S_out || !Vt_out || !ws) return dc_fail(DC_ERR_INVALID_ARG, "null pointer");
  if (dtype != DC_DTYPE_F32 && dtype != DC_DTYPE_BF16) return dc_fail(DC_ERR_INVALID_ARG, "dtype");
  if (d_out <= 0 || d_in <= 0 || r <= 0 || r > std::min(d_out, d_in))
    return dc_fail(DC_ERR_SHAPE, "rank %d outside 1..min(d_out, d_in)", r);
  if (oversample < 0 || power_iters < 0 || power_iters > 16) return dc_fail(DC_ERR_INVALID_ARG, "oversample / power_iters");
  if (((uintptr_t)ws & 255) != 0) return dc_fail(DC_ERR_ALIGN, "workspace must be 256-byte aligned");
  const void* ptrs[5] = {W_ft, W_base, U_out, S_out, Vt_out};
  for (const void* q : ptrs)
    if (((uintptr_t)q & 15) != 0) return dc_fail(DC_ERR_ALIGN, "device pointers must be 16-byte aligned");
  const int l = svd_l(d_out, d_in, r, oversample);
  const SvdWs W = svd_ws(d_out, d_in, l);
  if (ws_bytes < (size_t)W.total) return dc_fail(DC_ERR_WORKSPACE, "svd workspace holds %zu bytes, needs %lld", ws_bytes,
                                                 (long long)W.total);
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* b = (uint8_t*)ws;
  float* D = (float*)(b + W.delta);
  float* Qt = (float*)(b + W.qt);  // l x d_out: the columns of Y / Q
  float* Zt = (float*)(b + W.zt);  // l x d_in: Omega^T, then the columns of Z / B^T / W
  float* Jt = (float*)(b + W.jt);
  float* Ut = (float*)(b + W.ut);
  float* sig = (float*)(b + W.sig);
  double* G64 = (double*)(b + W.gram);
  float* Xinv = (float*)(b + W.tinv);
  int* off = (int*)(b + W.off);
  const float tol = 1e-6f;  // the final SVD's Jacobi tolerance
  const int max_sweeps = 40;
  int sweeps = 0;
  const int64_t nd = (int64_t)d_out * d_in;
  k_svd_delta<<<(unsigned)std::min<int64_t>((nd + 255) / 256, 148 * 32), 256, 0, s>>>(W_ft, W_base, dtype, D, nd);
  k_svd_gauss<<<(unsigned)std::min<int64_t>(((int64_t)l * d_in + 255) / 256, 148 * 32), 256, 0, s>>>(Zt, (int64_t)l * d_in, seed);
  dc_status st = dc_cuda_check(cudaGetLastError(), "svd setup");
  if (st) return st;
  // Y^T = Omega^T Delta^T, orth
  if ((st = gemm<true>(Zt, D, Qt, l, d_out, d_in, d_in, d_in, d_out, s))) return st;
  if ((st = orth_cholqr2(Qt, l, d_out, Ut, G64, Xinv, off, s))) return st;
  for (int it = 0; it < power_iters; ++it) {
    // Z^T = Q^T Delta (the columns of Delta^T Q), orth; Y^T = Z^T Delta^T, orth
    if ((st = gemm<false>(Qt, D, Zt, l, d_in, d_out, d_out, d_in, d_in, s))) return st;
    if ((st = orth_cholqr2(Zt, l, d_in, Ut, G64, Xinv, off, s))) return st;
    if ((st = gemm<true>(Zt, D, Qt, l, d_out, d_in, d_in, d_in, d_out, s))) return st;
    if ((st = orth_cholqr2(Qt, l, d_out, Ut, G64, Xinv, off, s))) return st;
  }
  // B^T = Delta^T Q (rows of Z^T), one-sided Jacobi with the rotations recorded in J
  if ((st = gemm<false>(Qt, D, Zt, l, d_in, d_out, d_out, d_in, d_in, s))) return st;
  k_identity<<<(unsigned)std::min<int64_t>(((int64_t)l * l + 255) / 256, 148 * 32), 256, 0, s>>>(Jt, l);
  if ((st = jacobi(Zt, l, d_in, Jt, tol, max_sweeps, off, s, &sweeps))) return st;
  k_row_norms<<<l, 256, 0, s>>>(Zt, d_in, sig, 0);
  // U^T = J^T Q^T: row j = u_j
  if ((st = gemm<false>(Jt, Qt, Ut, l, d_out, l, l, d_out, d_out, s))) return st;
  k_svd_emit<<<l, 256, 0, s>>>(sig, l, r, Zt, d_in, Ut, d_out, U_out, S_out, Vt_out);
  st = dc_cuda_check(cudaGetLastError(), "svd emit");
  if (st) return st;
  st = dc_cuda_check(cudaStreamSynchronize(s), "svd sync");
  if (st) return st;
  if (sweeps_out) *sweeps_out = sweeps;
  return DC_OK;
}
