// DVoRA (DoRA notes section 3.5): the direction update of VeRA,
// diag(b) B_shared diag(d) A_shared, inside DoRA. The layer is DoRA with
// B = B' = diag(b) B_shared diag(d) and A = A_shared, so the norm, forward,
// backward and merge calls run unchanged on B'; these kernels form B' and
// turn the gradient dB' into the gradients of the two trained vectors:
//   db[n] = sum_c dB'[n][c] B_shared[n][c] d[c]        (one warp per row)
//   dd[c] = sum_n dB'[n][c] b[n] B_shared[n][c]        (row-block partials,
//           then summed in block order: deterministic)
// All of it is a few passes over [d_out x r] values, bound by HBM.
#include <algorithm>

#include <cuda_bf16.h>

#include "dora_internal.h"

namespace dora {
namespace {

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// V elements of one row per access: 16 bytes for bf16 (whose rows are
// 16-byte aligned: r is a multiple of 8 and the tensors 16-byte aligned), one
// element for fp32 (only 4-byte alignment is required there).
template <class T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int V = 8;
  __device__ static void load(const __nv_bfloat16* p, float* f) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  __device__ static void store(__nv_bfloat16* p, const float* f) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = u;
  }
};
template <>
struct Vec<float> {
  static constexpr int V = 1;
  __device__ static void load(const float* p, float* f) { f[0] = *p; }
  __device__ static void store(float* p, const float* f) { *p = f[0]; }
};

template <class T>
__global__ void vera_compose_kernel(const T* __restrict__ Bs, const float* __restrict__ b,
                                    const float* __restrict__ d, int d_out, int r, T* __restrict__ Bp) {
  constexpr int V = Vec<T>::V;
  const int q = r / V;
  const long long total = (long long)d_out * q;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(i / q), c = (int)(i % q) * V;
    const long long off = (long long)n * r + c;
    float f[V];
    Vec<T>::load(Bs + off, f);
    const float bn = b[n];
#pragma unroll
    for (int j = 0; j < V; ++j) f[j] = bn * f[j] * d[c + j];
    Vec<T>::store(Bp + off, f);
  }
}

// One warp per row, V columns per lane and step.
template <class T>
__global__ void vera_db_kernel(const T* __restrict__ dBp, const T* __restrict__ Bs, const float* __restrict__ d,
                               int d_out, int r, float* __restrict__ db) {
  constexpr int V = Vec<T>::V;
  const int warps = blockDim.x / 32;
  const int lane = threadIdx.x & 31;
  for (int n = blockIdx.x * warps + (threadIdx.x >> 5); n < d_out; n += gridDim.x * warps) {
    float acc = 0.f;
#pragma unroll 2
    for (int c = lane * V; c < r; c += 32 * V) {
      const long long i = (long long)n * r + c;
      float g[V], w[V];
      Vec<T>::load(dBp + i, g);
      Vec<T>::load(Bs + i, w);
#pragma unroll
      for (int j = 0; j < V; ++j) acc = fmaf(g[j] * w[j], d[c + j], acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) db[n] = acc;
  }
}

// part[blk][c] = sum over rows [blk * rows, (blk + 1) * rows) of dB'[n][c] b[n] Bs[n][c]: each thread
// takes V columns of every (blockDim / (r / V))-th row of the block, then the row lanes are summed
// through shared memory in a fixed order.
template <class T>
__global__ void __launch_bounds__(256) vera_dd_partial_kernel(const T* __restrict__ dBp, const T* __restrict__ Bs,
                                                              const float* __restrict__ b, int d_out, int r,
                                                              int rows, float* __restrict__ part) {
  constexpr int V = Vec<T>::V;
  __shared__ float red[256 * V];
  const int q = r / V;  // column groups
  const int n0 = blockIdx.x * rows, n1 = min(d_out, n0 + rows);
  if (q > (int)blockDim.x) {
    // Rows wider than the block (fp32, r > 256): each thread sums whole columns.
    for (int c = threadIdx.x; c < r; c += blockDim.x) {
      float acc = 0.f;
      for (int n = n0; n < n1; ++n) {
        float g, w;
        Vec<T>::load(dBp + (long long)n * r + c, &g);
        Vec<T>::load(Bs + (long long)n * r + c, &w);
        acc = fmaf(g * w, b[n], acc);
      }
      part[(long long)blockIdx.x * r + c] = acc;
    }
    return;
  }
  const int lanes = (int)blockDim.x / q;  // row lanes, >= 1
  const int cg = threadIdx.x % q, rl = threadIdx.x / q;
  float acc[V];
#pragma unroll
  for (int j = 0; j < V; ++j) acc[j] = 0.f;
  if (rl < lanes) {
#pragma unroll 4
    for (int n = n0 + rl; n < n1; n += lanes) {
      const long long i = (long long)n * r + cg * V;
      float g[V], w[V];
      Vec<T>::load(dBp + i, g);
      Vec<T>::load(Bs + i, w);
      const float bn = b[n];
#pragma unroll
      for (int j = 0; j < V; ++j) acc[j] = fmaf(g[j] * w[j], bn, acc[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < V; ++j) red[threadIdx.x * V + j] = acc[j];
  __syncthreads();
  for (int c = threadIdx.x; c < r; c += blockDim.x) {
    const int g = c / V, j = c % V;
    float s = 0.f;
    for (int l = 0; l < lanes; ++l) s += red[(l * q + g) * V + j];
    part[(long long)blockIdx.x * r + c] = s;
  }
}

__global__ void vera_dd_final_kernel(const float* __restrict__ part, int nblk, int r, float* __restrict__ dd) {
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < r; c += gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int k = 0; k < nblk; ++k) acc += part[(long long)k * r + c];
    dd[c] = acc;
  }
}

template <class T>
cudaError_t vera_compose_t(const dora_desc_t& dsc, const void* Bs, const float* b, const float* d, void* Bp,
                           cudaStream_t st) {
  const long long total = dsc.d_out * (dsc.r / Vec<T>::V);
  ProfRange pr("vera_compose", st);
  vera_compose_kernel<T><<<(unsigned)std::min<long long>(cdiv(total, 256), 4096), 256, 0, st>>>(
      (const T*)Bs, b, d, (int)dsc.d_out, (int)dsc.r, (T*)Bp);
  return cudaGetLastError();
}

template <class T>
cudaError_t vera_grad_t(const dora_desc_t& dsc, const Plan& p, const void* Bs, const float* b, const float* d,
                        const void* dBp, float* db, float* dd, uint8_t* ws, cudaStream_t st) {
  const int d_out = (int)dsc.d_out, r = (int)dsc.r;
  {
    ProfRange pr("vera_db", st);
    vera_db_kernel<T><<<(unsigned)std::min<long long>(cdiv(d_out, 8), 1184), 256, 0, st>>>(
        (const T*)dBp, (const T*)Bs, d, d_out, r, db);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  float* part = reinterpret_cast<float*>(ws + p.off_f32_a);
  const int nblk = p.vera_blocks;
  const int rows = (int)cdiv(d_out, nblk);
  {
    ProfRange pr("vera_dd", st);
    vera_dd_partial_kernel<T><<<(unsigned)nblk, 256, 0, st>>>((const T*)dBp, (const T*)Bs, b, d_out, r, rows, part);
    vera_dd_final_kernel<<<(unsigned)cdiv(r, 256), 256, 0, st>>>(part, nblk, r, dd);
  }
  return cudaGetLastError();
}

}  // namespace

dora_status_t vera_compose(const dora_desc_t& dsc, const void* Bs, const float* b, const float* d, void* Bp,
                           cudaStream_t st) {
  const cudaError_t e = dsc.dtype == DORA_BF16 ? vera_compose_t<__nv_bfloat16>(dsc, Bs, b, d, Bp, st)
                                               : vera_compose_t<float>(dsc, Bs, b, d, Bp, st);
  return cuda_status(e, "dora_vera_compose");
}

dora_status_t vera_grad(const dora_desc_t& dsc, const Plan& p, const void* Bs, const float* b, const float* d,
                        const void* dBp, float* db, float* dd, uint8_t* ws, cudaStream_t st) {
  const cudaError_t e = dsc.dtype == DORA_BF16 ? vera_grad_t<__nv_bfloat16>(dsc, p, Bs, b, d, dBp, db, dd, ws, st)
                                               : vera_grad_t<float>(dsc, p, Bs, b, d, dBp, db, dd, ws, st);
  return cuda_status(e, "dora_vera_grad");
}

}  // namespace dora
