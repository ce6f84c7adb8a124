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

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <class T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

template <class T>
__global__ void vera_compose_kernel(const T* __restrict__ Bs, const float* __restrict__ b,
                                    const float* __restrict__ d, int d_out, int r, T* __restrict__ Bp) {
  const long long total = (long long)d_out * r;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(i / r), c = (int)(i % r);
    Bp[i] = from_f<T>(b[n] * to_f(Bs[i]) * d[c]);
  }
}

template <class T>
__global__ void vera_db_kernel(const T* __restrict__ dBp, const T* __restrict__ Bs, const float* __restrict__ d,
                               int d_out, int r, float* __restrict__ db) {
  const int warps = blockDim.x / 32;
  const int lane = threadIdx.x & 31;
  for (int n = blockIdx.x * warps + (threadIdx.x >> 5); n < d_out; n += gridDim.x * warps) {
    float acc = 0.f;
    for (int c = lane; c < r; c += 32) {
      const long long i = (long long)n * r + c;
      acc = fmaf(to_f(dBp[i]) * to_f(Bs[i]), d[c], acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) db[n] = acc;
  }
}

// part[blk][c] = sum over rows [blk * rows, (blk + 1) * rows) of dB'[n][c] b[n] Bs[n][c].
template <class T>
__global__ void vera_dd_partial_kernel(const T* __restrict__ dBp, const T* __restrict__ Bs,
                                       const float* __restrict__ b, int d_out, int r, int rows,
                                       float* __restrict__ part) {
  const int n0 = blockIdx.x * rows, n1 = min(d_out, n0 + rows);
  for (int c = threadIdx.x; c < r; c += blockDim.x) {
    float acc = 0.f;
    for (int n = n0; n < n1; ++n) {
      const long long i = (long long)n * r + c;
      acc = fmaf(to_f(dBp[i]) * to_f(Bs[i]), b[n], acc);
    }
    part[(long long)blockIdx.x * r + c] = acc;
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
  const long long total = dsc.d_out * dsc.r;
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
