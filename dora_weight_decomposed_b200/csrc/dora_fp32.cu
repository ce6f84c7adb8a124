// fp32 path of the DoRA layer on CUDA cores (FFMA). The tensor cores have no
// fp32 operand type that holds the 1e-4 norm tolerance (tf32 keeps 10 mantissa
// bits), so fp32 layers run the same factored math through SIMT kernels:
//
//   norm      P = W0 A^T, G = A A^T, Q = B G;  C_i^2 = |W0_i|^2 + 2 s B_i.P_i + s^2 B_i.Q_i
//   forward   su = s x A^T; pre = x W0^T + su B^T; y = pre + gm1 * pre
//   backward  dz = g * dy, dm = sum_t dy pre / C; du = s dz B; dB = dz^T su;
//             dA = du^T x; dx = dz W0 + du A
#include <algorithm>

#include "dora_internal.h"

namespace dora {

static inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// C[m][n] = alpha * sum_k A(m, k) B(n, k) + beta * C[m][n], with
// A(m, k) = A[m * sam + k * sak] and B(n, k) = B[n * sbn + k * sbk].
// 64 x 64 tile, 16-deep K slices, 4 x 4 outputs per thread.
__global__ void __launch_bounds__(256) sgemm_strided_kernel(int M, int N, int K, const float* __restrict__ A,
                                                            long long sam, long long sak,
                                                            const float* __restrict__ B, long long sbn,
                                                            long long sbk, float* __restrict__ C, long long ldc,
                                                            float alpha, float beta) {
  __shared__ float As[16][65];
  __shared__ float Bs[16][65];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 16 * 64; i += 256) {
      const int kk = i >> 6, mm = i & 63;
      const int k = k0 + kk;
      As[kk][mm] = (m0 + mm < M && k < K) ? A[(long long)(m0 + mm) * sam + (long long)k * sak] : 0.f;
      Bs[kk][mm] = (n0 + mm < N && k < K) ? B[(long long)(n0 + mm) * sbn + (long long)k * sbk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float* c = C + (long long)m * ldc + n;
      *c = beta != 0.f ? fmaf(alpha, acc[i][j], beta * *c) : alpha * acc[i][j];
    }
  }
}

static cudaError_t sgemm(int M, int N, int K, const float* A, long long sam, long long sak, const float* B,
                         long long sbn, long long sbk, float* C, long long ldc, float alpha, float beta,
                         cudaStream_t st) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((unsigned)cdiv(N, 64), (unsigned)cdiv(M, 64));
  ProfRange pr("sgemm", st);
  sgemm_strided_kernel<<<grid, 256, 0, st>>>(M, N, std::max(K, 0), A, sam, sak, B, sbn, sbk, C, ldc, alpha, beta);
  return cudaGetLastError();
}

// One warp per row: C_i^2 = |W0_i|^2 + 2 s B_i.P_i + s^2 B_i.Q_i, then C, g, g - 1.
__global__ void f32_norm_rows_kernel(const float* __restrict__ W0, const float* __restrict__ B,
                                     const float* __restrict__ P, const float* __restrict__ Q,
                                     const float* __restrict__ m, int d_out, int d_in, int r, float s,
                                     float* __restrict__ C, float* __restrict__ g, float* __restrict__ gm1) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= d_out) return;
  float ss = 0.f, cross = 0.f, gram = 0.f;
  for (int k = lane; k < d_in; k += 32) {
    const float w = W0[(long long)row * d_in + k];
    ss = fmaf(w, w, ss);
  }
  for (int n = lane; n < r; n += 32) {
    const float b = B[(long long)row * r + n];
    cross = fmaf(b, P[(long long)row * r + n], cross);
    gram = fmaf(b, Q[(long long)row * r + n], gram);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    cross += __shfl_xor_sync(0xffffffffu, cross, o);
    gram += __shfl_xor_sync(0xffffffffu, gram, o);
  }
  if (lane == 0) {
    const float sq = ss + 2.f * s * cross + s * s * gram;
    const float c = sqrtf(fmaxf(sq, 0.f));
    const float mi = m[row];
    C[row] = c;
    g[row] = mi / c;
    gm1[row] = (mi - c) / c;
  }
}

// y = pre + gm1[n] * pre over [T x d_out].
__global__ void f32_compose_kernel(const float* __restrict__ pre, const float* __restrict__ gm1,
                                   float* __restrict__ y, long long total, int d_out) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const float v = pre[i];
    y[i] = fmaf(gm1[i % d_out], v, v);
  }
}

// dz = g * dy; part[rb][i] = sum over the row block of dy * pre. Thread per column.
constexpr int kF32Rows = 64;

__global__ void f32_compose_bwd_kernel(const float* __restrict__ dy, const float* __restrict__ pre,
                                       const float* __restrict__ g, float* __restrict__ dz,
                                       float* __restrict__ part, int T, int d_out) {
  const int col = blockIdx.x * blockDim.x + threadIdx.x;
  if (col >= d_out) return;
  const int t0 = blockIdx.y * kF32Rows, t1 = min(T, t0 + kF32Rows);
  const float gc = g[col];
  float acc = 0.f;
  for (int t = t0; t < t1; ++t) {
    const long long off = (long long)t * d_out + col;
    const float a = dy[off];
    acc = fmaf(a, pre[off], acc);
    dz[off] = gc * a;
  }
  part[(long long)blockIdx.y * d_out + col] = acc;
}

__global__ void f32_dm_finalize_kernel(const float* __restrict__ part, int nparts, int d_out,
                                       const float* __restrict__ C, float* __restrict__ dm) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= d_out) return;
  float s = 0.f;
  for (int z = 0; z < nparts; ++z) s += part[(long long)z * d_out + i];
  dm[i] = s / C[i];
}

// W_out[i][j] = g_i (W0[i][j] + s sum_k B[i][k] A[k][j]); one thread per element.
__global__ void f32_merge_kernel(const float* __restrict__ W0, const float* __restrict__ A,
                                 const float* __restrict__ B, const float* __restrict__ g, float* W_out, int d_out,
                                 int d_in, int r, float s) {
  const long long total = (long long)d_out * d_in;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(e / d_in), j = (int)(e % d_in);
    float acc = 0.f;
    for (int k = 0; k < r; ++k) acc = fmaf(B[(long long)i * r + k], A[(long long)k * d_in + j], acc);
    W_out[e] = g[i] * fmaf(s, acc, W0[e]);
  }
}

dora_status_t f32_merge(const dora_desc_t& d, const float* W0, const float* A, const float* B, const float* g,
                        float* W_out, cudaStream_t st) {
  const long long total = d.d_out * d.d_in;
  ProfRange pr("f32_merge", st);
  f32_merge_kernel<<<(unsigned)std::min<long long>(cdiv(total, 256), 4096), 256, 0, st>>>(
      W0, A, B, g, W_out, (int)d.d_out, (int)d.d_in, (int)d.r, d.s);
  return cuda_status(cudaGetLastError(), "dora_merge (fp32)");
}

dora_status_t f32_norm(const dora_desc_t& d, const Plan& p, const float* W0, const float* A, const float* B,
                       const float* m, float* C, float* g, float* gm1, uint8_t* ws, cudaStream_t st) {
  const int r = (int)d.r, d_in = (int)d.d_in, d_out = (int)d.d_out;
  float* P = reinterpret_cast<float*>(ws + p.off_f32_a);
  float* G = reinterpret_cast<float*>(ws + p.off_f32_b);
  float* Q = reinterpret_cast<float*>(ws + p.off_f32_c);
  cudaError_t e = sgemm(d_out, r, d_in, W0, d_in, 1, A, d_in, 1, P, r, 1.f, 0.f, st);   // P = W0 A^T
  if (e == cudaSuccess) e = sgemm(r, r, d_in, A, d_in, 1, A, d_in, 1, G, r, 1.f, 0.f, st);  // G = A A^T
  if (e == cudaSuccess) e = sgemm(d_out, r, r, B, r, 1, G, r, 1, Q, r, 1.f, 0.f, st);      // Q = B G
  if (e != cudaSuccess) return cuda_status(e, "dora_norm (fp32)");
  ProfRange pr("f32_norm_rows", st);
  f32_norm_rows_kernel<<<(unsigned)cdiv(d_out, 8), 256, 0, st>>>(W0, B, P, Q, m, d_out, d_in, r, d.s, C, g, gm1);
  return cuda_status(cudaGetLastError(), "dora_norm (fp32)");
}

dora_status_t f32_forward(const dora_desc_t& d, const Plan& p, int64_t T, const float* x, const float* W0,
                          const float* A, const float* B, const float* gm1, float* y, float* su_save,
                          float* pre_save, uint8_t* ws, cudaStream_t st) {
  if (T == 0) return DORA_OK;
  const int r = (int)d.r, d_in = (int)d.d_in, d_out = (int)d.d_out, Ti = (int)T;
  float* su = su_save ? su_save : reinterpret_cast<float*>(ws + p.off_f32_a);
  float* pre = pre_save ? pre_save : reinterpret_cast<float*>(ws + p.off_f32_b);
  cudaError_t e = sgemm(Ti, r, d_in, x, d_in, 1, A, d_in, 1, su, r, d.s, 0.f, st);               // su = s x A^T
  if (e == cudaSuccess) e = sgemm(Ti, d_out, d_in, x, d_in, 1, W0, d_in, 1, pre, d_out, 1.f, 0.f, st);  // x W0^T
  if (e == cudaSuccess) e = sgemm(Ti, d_out, r, su, r, 1, B, r, 1, pre, d_out, 1.f, 1.f, st);          // + su B^T
  if (e != cudaSuccess) return cuda_status(e, "dora_forward (fp32)");
  const long long total = (long long)Ti * d_out;
  ProfRange pr("f32_compose", st);
  f32_compose_kernel<<<(unsigned)std::min<long long>(cdiv(total, 256), 4096), 256, 0, st>>>(pre, gm1, y, total,
                                                                                            d_out);
  return cuda_status(cudaGetLastError(), "dora_forward (fp32)");
}

dora_status_t f32_backward(const dora_desc_t& d, const Plan& p, int64_t T, const float* dy, const float* x,
                           const float* W0, const float* A, const float* B, const float* C, const float* g,
                           const float* su, const float* pre, float* dm, float* dA, float* dB, float* dx,
                           uint8_t* ws, cudaStream_t st) {
  const int r = (int)d.r, d_in = (int)d.d_in, d_out = (int)d.d_out, Ti = (int)T;
  if (T == 0) {
    cudaError_t e = cudaMemsetAsync(dm, 0, sizeof(float) * d_out, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dA, 0, sizeof(float) * r * d_in, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dB, 0, sizeof(float) * d_out * r, st);
    return cuda_status(e, "dora_backward (fp32): empty batch");
  }
  float* dz = reinterpret_cast<float*>(ws + p.off_f32_a);
  float* part = reinterpret_cast<float*>(ws + p.off_f32_b);
  float* du = reinterpret_cast<float*>(ws + p.off_f32_c);
  const int rb = (int)cdiv(Ti, kF32Rows);
  {
    ProfRange pr("f32_compose_bwd", st);
    f32_compose_bwd_kernel<<<dim3((unsigned)cdiv(d_out, 128), (unsigned)rb), 128, 0, st>>>(dy, pre, g, dz, part,
                                                                                           Ti, d_out);
  }
  {
    ProfRange pr("f32_dm_finalize", st);
    f32_dm_finalize_kernel<<<(unsigned)cdiv(d_out, 256), 256, 0, st>>>(part, rb, d_out, C, dm);
  }
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = sgemm(Ti, r, d_out, dz, d_out, 1, B, 1, r, du, r, d.s, 0.f, st);      // du = s dz B
  if (e == cudaSuccess) e = sgemm(d_out, r, Ti, dz, 1, d_out, su, 1, r, dB, r, 1.f, 0.f, st);     // dB = dz^T su
  if (e == cudaSuccess) e = sgemm(r, d_in, Ti, du, 1, r, x, 1, d_in, dA, d_in, 1.f, 0.f, st);     // dA = du^T x
  if (e == cudaSuccess && dx) {
    e = sgemm(Ti, d_in, d_out, dz, d_out, 1, W0, 1, d_in, dx, d_in, 1.f, 0.f, st);                 // dx = dz W0
    if (e == cudaSuccess) e = sgemm(Ti, d_in, r, du, r, 1, A, 1, d_in, dx, d_in, 1.f, 1.f, st);   //    + du A
  }
  return cuda_status(e, "dora_backward (fp32)");
}

}  // namespace dora

namespace dora {

// kappa_n = g_n dm_n / C_n and Bk[n][c] = kappa_n B[n][c].
__global__ void f32_kappa_kernel(const float* __restrict__ g, const float* __restrict__ dm,
                                 const float* __restrict__ C, const float* __restrict__ B, int d_out, int r,
                                 float* __restrict__ kappa, float* __restrict__ Bk) {
  const long long total = (long long)d_out * r;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(i / r), c = (int)(i % r);
    const float k = g[n] * dm[n] / C[n];
    if (c == 0) kappa[n] = k;
    Bk[i] = k * B[i];
  }
}

// dB[n][c] -= s kappa_n Q[n][c].
__global__ void f32_full_dB_kernel(const float* __restrict__ Q, const float* __restrict__ kappa, int d_out, int r,
                                   float s, float* __restrict__ dB) {
  const long long total = (long long)d_out * r;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x)
    dB[i] = fmaf(-s * kappa[i / r], Q[i], dB[i]);
}

// Full (non-detached) gradient, fp32: the detached backward, then
//   dB -= s diag(kappa) (W0 A^T + s B G),  G = A A^T
//   dA -= s (kappa B)^T W0 + s^2 (B^T diag(kappa) B) A
dora_status_t f32_backward_full(const dora_desc_t& d, const Plan& p, int64_t T, const float* dy, const float* x,
                                const float* W0, const float* A, const float* B, const float* C, const float* g,
                                const float* su, const float* pre, float* dm, float* dA, float* dB, float* dx,
                                uint8_t* ws, cudaStream_t st) {
  dora_status_t status = f32_backward(d, p, T, dy, x, W0, A, B, C, g, su, pre, dm, dA, dB, dx, ws, st);
  if (status != DORA_OK || T == 0) return status;  // no tokens: dm = 0, so kappa = 0
  const int r = (int)d.r, d_in = (int)d.d_in, d_out = (int)d.d_out;
  float* kappa = reinterpret_cast<float*>(ws + p.off_kappa);
  float* Bk = reinterpret_cast<float*>(ws + p.off_bk);
  float* G = reinterpret_cast<float*>(ws + p.off_gs);
  float* Q = reinterpret_cast<float*>(ws + p.off_q_part);
  float* H = reinterpret_cast<float*>(ws + p.off_h);
  const long long n = (long long)d_out * r;
  {
    ProfRange pr("f32_full_kappa", st);
    f32_kappa_kernel<<<(unsigned)std::min<long long>(cdiv(n, 256), 4096), 256, 0, st>>>(g, dm, C, B, d_out, r, kappa,
                                                                                         Bk);
  }
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = sgemm(r, r, d_in, A, d_in, 1, A, d_in, 1, G, r, 1.f, 0.f, st);            // G = A A^T
  if (e == cudaSuccess) e = sgemm(d_out, r, d_in, W0, d_in, 1, A, d_in, 1, Q, r, 1.f, 0.f, st);       // Q = W0 A^T
  if (e == cudaSuccess) e = sgemm(d_out, r, r, B, r, 1, G, r, 1, Q, r, d.s, 1.f, st);                 //   + s B G
  if (e == cudaSuccess) {
    ProfRange pr("f32_full_dB", st);
    f32_full_dB_kernel<<<(unsigned)std::min<long long>(cdiv(n, 256), 4096), 256, 0, st>>>(Q, kappa, d_out, r, d.s,
                                                                                           dB);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = sgemm(r, r, d_out, Bk, 1, r, B, 1, r, H, r, 1.f, 0.f, st);                 // H = (kB)^T B
  if (e == cudaSuccess) e = sgemm(r, d_in, d_out, Bk, 1, r, W0, 1, d_in, dA, d_in, -d.s, 1.f, st);     // dA -= s (kB)^T W0
  if (e == cudaSuccess) e = sgemm(r, d_in, r, H, r, 1, A, 1, d_in, dA, d_in, -d.s * d.s, 1.f, st);     //    - s^2 H A
  return cuda_status(e, "dora_backward_full (fp32)");
}

}  // namespace dora
