// Shard-layout kernels: bit-exact copies between the unsharded weight layout
// and the shard-packed one ("How transformer layers actually decompose":
// W1 split by columns as [W1_left | W1_right], W2 split by rows as
// [W2_top; W2_bottom]; "The attention heads split": Q, K, V split by the
// columns of each shard's heads).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "internal.h"

namespace tp {

namespace {

// Packed element e of [t][rows][ct]  <->  full element (r, i*ct + c) of [rows][t*ct].
template <int V>
__global__ void shard_cols_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst,
                                  long long rows, long long ct, int t, bool inverse) {
  const long long per = rows * ct;
  const long long n = per * t / V;
  for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < n;
       v += (long long)gridDim.x * blockDim.x) {
    const long long e = v * V;
    const long long i = e / per;
    const long long rem = e - i * per;
    const long long r = rem / ct;
    const long long c = rem - r * ct;
    const long long full = r * ct * t + i * ct + c;
    if (V == 8) {
      if (inverse)
        *reinterpret_cast<uint4*>(dst + full) = *reinterpret_cast<const uint4*>(src + e);
      else
        *reinterpret_cast<uint4*>(dst + e) = *reinterpret_cast<const uint4*>(src + full);
    } else {
      if (inverse) dst[full] = src[e];
      else dst[e] = src[full];
    }
  }
}

// Packed element e of [t][rows][3dt]  <->  full element (r, j*D + i*dt + c) of [rows][3D].
template <int V>
__global__ void shard_qkv_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst,
                                 long long rows, long long dt, int t, bool inverse) {
  const long long w3 = 3 * dt;
  const long long per = rows * w3;
  const long long n = per * t / V;
  const long long D = dt * t;
  for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < n;
       v += (long long)gridDim.x * blockDim.x) {
    const long long e = v * V;
    const long long i = e / per;
    const long long rem = e - i * per;
    const long long r = rem / w3;
    const long long cc = rem - r * w3;
    const long long j = cc / dt;
    const long long c = cc - j * dt;
    const long long full = r * 3 * D + j * D + i * dt + c;
    if (V == 8) {
      if (inverse)
        *reinterpret_cast<uint4*>(dst + full) = *reinterpret_cast<const uint4*>(src + e);
      else
        *reinterpret_cast<uint4*>(dst + e) = *reinterpret_cast<const uint4*>(src + full);
    } else {
      if (inverse) dst[full] = src[e];
      else dst[e] = src[full];
    }
  }
}

template <int V>
__global__ void copy_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst,
                            long long n) {
  for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < n / V;
       v += (long long)gridDim.x * blockDim.x) {
    if (V == 8) *reinterpret_cast<uint4*>(dst + v * 8) = *reinterpret_cast<const uint4*>(src + v * 8);
    else dst[v] = src[v];
  }
}

// bf16 -> fp16, 8 elements per thread step, four steps' loads issued before
// their conversions; out-of-range values flag `err`.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4 u, bool& over) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  uint32_t o[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float lo = __uint_as_float(w[q] << 16), hi = __uint_as_float(w[q] & 0xFFFF0000u);
    over |= fabsf(lo) > 65504.0f || fabsf(hi) > 65504.0f;
    __half2 h = __floats2half2_rn(lo, hi);
    o[q] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__global__ void cast_f16_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst,
                                long long n8, unsigned int* err) {
  grid_dep_wait();
  grid_dep_launch();
  bool over = false;
  const long long stride = (long long)gridDim.x * blockDim.x;
  long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  for (; v + 3 * stride < n8; v += 4 * stride) {
    uint4 u[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) u[j] = *reinterpret_cast<const uint4*>(src + (v + j * stride) * 8);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<uint4*>(dst + (v + j * stride) * 8) = bf16x8_to_f16x8(u[j], over);
  }
  for (; v < n8; v += stride)
    *reinterpret_cast<uint4*>(dst + v * 8) =
        bf16x8_to_f16x8(*reinterpret_cast<const uint4*>(src + v * 8), over);
  if (over && err) atomicCAS(err, 0u, 0x301u);
}

int grid_for(long long work) {
  const long long cap = (long long)sm_count() * 8;
  long long g = (work + 255) / 256;
  if (g > cap) g = cap;
  return g < 1 ? 1 : (int)g;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

tp_status launch_shard_cols(const uint16_t* src, int rows, int cols, int t, uint16_t* dst,
                            bool inverse, cudaStream_t stream) {
  const long long ct = cols / t;
  const long long n = (long long)rows * cols;
  if (n == 0) return TP_OK;
  TraceScope ts(stream, TK_LAYOUT);
  if (ct % 8 == 0 && aligned16(src) && aligned16(dst))
    shard_cols_kernel<8><<<grid_for(n / 8), 256, 0, stream>>>(src, dst, rows, ct, t, inverse);
  else
    shard_cols_kernel<1><<<grid_for(n), 256, 0, stream>>>(src, dst, rows, ct, t, inverse);
  return cuda_status(cudaGetLastError());
}

tp_status launch_shard_qkv(const uint16_t* src, int rows, int hidden, int t, uint16_t* dst,
                           bool inverse, cudaStream_t stream) {
  const long long dt = hidden / t;
  const long long n = (long long)rows * 3 * hidden;
  if (n == 0) return TP_OK;
  TraceScope ts(stream, TK_LAYOUT);
  if (dt % 8 == 0 && aligned16(src) && aligned16(dst))
    shard_qkv_kernel<8><<<grid_for(n / 8), 256, 0, stream>>>(src, dst, rows, dt, t, inverse);
  else
    shard_qkv_kernel<1><<<grid_for(n), 256, 0, stream>>>(src, dst, rows, dt, t, inverse);
  return cuda_status(cudaGetLastError());
}

tp_status launch_copy(const uint16_t* src, size_t n, uint16_t* dst, cudaStream_t stream) {
  if (n == 0) return TP_OK;
  TraceScope ts(stream, TK_LAYOUT);
  if (n % 8 == 0 && aligned16(src) && aligned16(dst))
    copy_kernel<8><<<grid_for((long long)n / 8), 256, 0, stream>>>(src, dst, (long long)n);
  else
    copy_kernel<1><<<grid_for((long long)n), 256, 0, stream>>>(src, dst, (long long)n);
  return cuda_status(cudaGetLastError());
}

tp_status launch_cast_f16(const uint16_t* src, size_t n, uint16_t* dst, cudaStream_t stream) {
  if (n == 0) return TP_OK;
  if (n % 8 || !aligned16(src) || !aligned16(dst)) return TP_ERR_MISALIGNED;
  TraceScope ts(stream, TK_CAST);
  if (launch_pdl(cast_f16_kernel, dim3(grid_for((long long)n / 8)), dim3(256), 0, stream, src, dst,
                 (long long)n / 8, error_word()) != cudaSuccess)
    return TP_ERR_CUDA;
  return cuda_status(cudaGetLastError());
}

}  // namespace tp
