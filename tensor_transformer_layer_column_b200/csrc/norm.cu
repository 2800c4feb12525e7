// HBM-bound row and column kernels: LayerNorm forward / backward (pre-LN,
// "The layernorm placement the paper flags as critical") and deterministic
// column sums for bias gradients.  128-bit loads and stores throughout; fp32
// statistics; every reduction order is fixed, so results repeat bit for bit.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "internal.h"

namespace tp {

namespace {

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    f[2 * q] = __uint_as_float(w[q] << 16);
    f[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 u;
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __nv_bfloat162 v = __floats2bfloat162_rn(f[2 * q], f[2 * q + 1]);
    w[q] = *reinterpret_cast<uint32_t*>(&v);
  }
  u.x = w[0]; u.y = w[1]; u.z = w[2]; u.w = w[3];
  return u;
}

__device__ __forceinline__ void unpack8_f16(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __half2 h = *reinterpret_cast<const __half2*>(&w[q]);
    const float2 v = __half22float2(h);
    f[2 * q] = v.x;
    f[2 * q + 1] = v.y;
  }
}

__device__ __forceinline__ uint4 pack8_f16(const float (&f)[8]) {
  uint4 u;
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __half2 v = __floats2half2_rn(f[2 * q], f[2 * q + 1]);
    w[q] = *reinterpret_cast<uint32_t*>(&v);
  }
  u.x = w[0]; u.y = w[1]; u.z = w[2]; u.w = w[3];
  return u;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One warp per row, rows walked grid-stride; lane owns 8-element chunks lane,
// lane+32, ...  The row stays in registers as packed bf16 (4 registers per
// chunk), so two 256-thread blocks fit per SM.  Statistics in fp32, two
// passes over the registers (mean, then centred variance).  The output is
// bf16, or fp16 when F16OUT (values beyond the fp16 range set `err` to 0x301).
template <int CH, bool F16OUT>
__global__ void __launch_bounds__(256, 2)
ln_fwd_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ g,
              const uint16_t* __restrict__ b, long long rows, int D, float eps,
              uint16_t* __restrict__ y, float* __restrict__ mean, float* __restrict__ rstd,
              unsigned int* err) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int nch = D >> 3;
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  bool over = false;
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += nwarps) {
    const uint16_t* xr = x + row * D;
    uint4 pk[CH];
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      const int c = lane + 32 * j;
      if (c < nch) pk[j] = *reinterpret_cast<const uint4*>(xr + c * 8);
    }
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      if (lane + 32 * j < nch) {
        float v[8];
        unpack8(pk[j], v);
#pragma unroll
        for (int e = 0; e < 8; ++e) s += v[e];
      }
    }
    const float mu = warp_sum(s) / D;
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      if (lane + 32 * j < nch) {
        float v[8];
        unpack8(pk[j], v);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float d = v[e] - mu;
          ss += d * d;
        }
      }
    }
    const float rs = rsqrtf(warp_sum(ss) / D + eps);
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      const int c = lane + 32 * j;
      if (c < nch) {
        float v[8], gv[8], bv[8], o[8];
        unpack8(pk[j], v);
        unpack8(*reinterpret_cast<const uint4*>(g + c * 8), gv);
        unpack8(*reinterpret_cast<const uint4*>(b + c * 8), bv);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = (v[e] - mu) * rs * gv[e] + bv[e];
        if (F16OUT) {
          *reinterpret_cast<uint4*>(y + row * D + c * 8) = pack8_f16(o);
#pragma unroll
          for (int e = 0; e < 8; ++e) over |= fabsf(o[e]) > 65504.0f;
        } else {
          *reinterpret_cast<uint4*>(y + row * D + c * 8) = pack8(o);
        }
      }
    }
    if (lane == 0) {
      mean[row] = mu;
      rstd[row] = rs;
    }
  }
  if (F16OUT && over && err) atomicCAS(err, 0u, 0x301u);
}

constexpr int LNB_THREADS = 256;

// One block walks a contiguous chunk of rows; thread owns 8-element chunks
// tid, tid+256, ...; the next row's operands are loaded while the current
// row goes through its block reduction.  Per-block dgamma/dbeta partials go to
// `partial` [gridDim.x][2][D] and are reduced by ln_param_reduce in block order.
// Eight consecutive elements of the upstream gradient, bf16 or fp32.
template <bool F32>
struct DyChunk {
  uint4 v;
  __device__ __forceinline__ void load(const void* p, long long off) {
    v = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p) + off);
  }
  __device__ __forceinline__ void get(float (&o)[8]) const { unpack8(v, o); }
};
template <>
struct DyChunk<true> {
  float4 a, b;
  __device__ __forceinline__ void load(const void* p, long long off) {
    const float* q = static_cast<const float*>(p) + off;
    a = *reinterpret_cast<const float4*>(q);
    b = *reinterpret_cast<const float4*>(q + 4);
  }
  __device__ __forceinline__ void get(float (&o)[8]) const {
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  }
};

// DY32: dy is fp32.  dx32, when set, receives an fp32 copy of dx.  RSUM: the
// block also sums the rows of dres (a third partial row, [gridDim.x][3][D]):
// the column sums of a residual gradient that passes through, e.g. the bias
// gradient of the row-parallel product that produced it.
template <int CH, bool DY32 = false, bool RSUM = false>
__global__ void __launch_bounds__(LNB_THREADS, 2)
ln_bwd_kernel(const void* __restrict__ dy, const uint16_t* __restrict__ x,
              const uint16_t* __restrict__ g, const float* __restrict__ mean,
              const float* __restrict__ rstd, const uint16_t* __restrict__ dres, long long rows,
              int D, int rows_per_block, uint16_t* __restrict__ dx, float* __restrict__ partial,
              float* __restrict__ dx32 = nullptr) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ float red[2][2][LNB_THREADS / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nch = D >> 3;
  // gamma stays packed (bf16); xhat and g = dy * gamma are recomputed from the
  // packed row in the output pass instead of being held in fp32 registers.
  uint4 gpk[CH];
  float adg[CH][8], adb[CH][8], adr[RSUM ? CH : 1][8];
#pragma unroll
  for (int j = 0; j < CH; ++j) {
    const int c = tid + LNB_THREADS * j;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      adg[j][e] = adb[j][e] = 0.f;
      if (RSUM) adr[j][e] = 0.f;
    }
    if (c < nch) gpk[j] = *reinterpret_cast<const uint4*>(g + c * 8);
  }
  const long long r0 = (long long)blockIdx.x * rows_per_block;
  const long long r1 = min(rows, r0 + rows_per_block);
  const float invD = 1.0f / D;
  DyChunk<DY32> cdy[CH];
  uint4 cx[CH], cres[CH];
  auto load_row = [&](long long r, DyChunk<DY32> (&ody)[CH], uint4 (&ox)[CH], uint4 (&ores)[CH]) {
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      const int c = tid + LNB_THREADS * j;
      if (c < nch) {
        ody[j].load(dy, r * D + c * 8);
        ox[j] = *reinterpret_cast<const uint4*>(x + r * D + c * 8);
        if (dres != nullptr) ores[j] = *reinterpret_cast<const uint4*>(dres + r * D + c * 8);
      }
    }
  };
  if (r0 < r1) load_row(r0, cdy, cx, cres);
  int buf = 0;
  for (long long r = r0; r < r1; ++r, buf ^= 1) {
    DyChunk<DY32> ndy[CH];
    uint4 nx[CH], nres[CH];
    if (r + 1 < r1) load_row(r + 1, ndy, nx, nres);
    const float mu = mean[r], rs = rstd[r];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      if (tid + LNB_THREADS * j < nch) {
        float dv[8], xv[8], gm[8];
        cdy[j].get(dv);
        unpack8(cx[j], xv);
        unpack8(gpk[j], gm);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float xh = (xv[e] - mu) * rs;
          const float gv = dv[e] * gm[e];
          s1 += gv;
          s2 += gv * xh;
          adg[j][e] += dv[e] * xh;
          adb[j][e] += dv[e];
        }
      }
    }
    s1 = warp_sum(s1);
    s2 = warp_sum(s2);
    if (lane == 0) {
      red[buf][0][warp] = s1;
      red[buf][1][warp] = s2;
    }
    __syncthreads();
    s1 = 0.f;
    s2 = 0.f;
#pragma unroll
    for (int w = 0; w < LNB_THREADS / 32; ++w) {
      s1 += red[buf][0][w];
      s2 += red[buf][1][w];
    }
    const float m1 = s1 * invD, m2 = s2 * invD;
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      const int c = tid + LNB_THREADS * j;
      if (c < nch) {
        float dv[8], xv[8], gm[8], o[8];
        cdy[j].get(dv);
        unpack8(cx[j], xv);
        unpack8(gpk[j], gm);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float xh = (xv[e] - mu) * rs;
          o[e] = rs * (dv[e] * gm[e] - m1 - xh * m2);
        }
        if (dres != nullptr) {
          float rv[8];
          unpack8(cres[j], rv);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            o[e] += rv[e];
            if (RSUM) adr[j][e] += rv[e];
          }
        }
        *reinterpret_cast<uint4*>(dx + r * D + c * 8) = pack8(o);
        if (dx32 != nullptr) {
          float* q = dx32 + r * D + c * 8;
          *reinterpret_cast<float4*>(q) = make_float4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<float4*>(q + 4) = make_float4(o[4], o[5], o[6], o[7]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      cdy[j] = ndy[j];
      cx[j] = nx[j];
      cres[j] = nres[j];
    }
  }
  float* pg = partial + (long long)blockIdx.x * (RSUM ? 3 : 2) * D;
#pragma unroll
  for (int j = 0; j < CH; ++j) {
    const int c = tid + LNB_THREADS * j;
    if (c < nch) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        pg[c * 8 + e] = adg[j][e];
        pg[D + c * 8 + e] = adb[j][e];
        if (RSUM) pg[2 * D + c * 8 + e] = adr[j][e];
      }
    }
  }
}

// Fixed-order reduction of `n` partial rows of `width` floats: block x covers
// 32 columns; warp w sums rows w, w+8, ... of its column (coalesced 128-byte
// rows), then warp 0 adds the 8 warp sums in order.  Returns the total for
// column blockIdx.x*32 + lane in warp 0 (valid when that column exists).
__device__ __forceinline__ float reduce_rows_fixed(const float* __restrict__ rowsrc, int n,
                                                   long long width, long long stride_rows,
                                                   float (*red)[33]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long c = (long long)blockIdx.x * 32 + lane;
  float s = 0.f;
  if (c < width) {
    // Eight rows' loads issued ahead of their (in-order) additions.
    int k = warp;
    for (; k + 56 < n; k += 64) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = rowsrc[(long long)(k + 8 * j) * stride_rows + c];
#pragma unroll
      for (int j = 0; j < 8; ++j) s += v[j];
    }
    for (; k < n; k += 8) s += rowsrc[(long long)k * stride_rows + c];
  }
  red[warp][lane] = s;
  __syncthreads();
  float t = 0.f;
  if (warp == 0) {
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w][lane];
  }
  return t;
}

// out_k[c] = sum over blocks b (fixed order) of partial[b][k][c], k < nk:
// 0 dgamma, 1 dbeta, 2 the column sums of dres.
__global__ void __launch_bounds__(256)
ln_param_reduce(const float* __restrict__ partial, int nblocks, int D, int nk,
                uint16_t* __restrict__ dg, uint16_t* __restrict__ db, uint16_t* __restrict__ dr) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ float red[8][33];
  const long long width = (long long)nk * D;
  const float t = reduce_rows_fixed(partial, nblocks, width, width, red);
  const int i = blockIdx.x * 32 + (threadIdx.x & 31);
  if ((threadIdx.x >> 5) != 0 || i >= width) return;
  const int k = i / D;
  uint16_t* out = k == 0 ? dg : (k == 1 ? db : dr);
  if (out == nullptr) return;
  __nv_bfloat16 v = __float2bfloat16_rn(t);
  out[i - k * D] = *reinterpret_cast<uint16_t*>(&v);
}

// Column sums of S stacked [rows][cols] matrices, pass 1: block (cx, cy, s)
// sums rows [cy*rpc, (cy+1)*rpc) of columns [cx*2048, cx*2048+2048) of matrix s,
// four rows in flight per thread.
template <bool F16IN>
__global__ void __launch_bounds__(256)
colsum_partial_kernel(const uint16_t* __restrict__ x, long long rows, long long cols,
                      int rows_per_chunk, float* __restrict__ partial) {
  const long long c = ((long long)blockIdx.x * 256 + threadIdx.x) * 8;
  if (c >= cols) return;
  const long long s = blockIdx.z;
  const long long r0 = (long long)blockIdx.y * rows_per_chunk;
  const long long r1 = min(rows, r0 + rows_per_chunk);
  const uint16_t* base = x + s * rows * cols + c;
  float acc[4][8];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[u][e] = 0.f;
  long long r = r0;
  for (; r + 4 <= r1; r += 4) {
    uint4 q[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) q[u] = *reinterpret_cast<const uint4*>(base + (r + u) * cols);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float v[8];
      if (F16IN) unpack8_f16(q[u], v);
      else unpack8(q[u], v);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[u][e] += v[e];
    }
  }
  for (; r < r1; ++r) {
    float v[8];
    if (F16IN) unpack8_f16(*reinterpret_cast<const uint4*>(base + r * cols), v);
    else unpack8(*reinterpret_cast<const uint4*>(base + r * cols), v);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[0][e] += v[e];
  }
  float* p = partial + (s * gridDim.y + blockIdx.y) * cols + c;
#pragma unroll
  for (int e = 0; e < 8; ++e) p[e] = (acc[0][e] + acc[1][e]) + (acc[2][e] + acc[3][e]);
}

// Pass 2: out[s][c] = sum over chunks k (fixed order) of partial[s][k][c].
__global__ void __launch_bounds__(256)
colsum_reduce_kernel(const float* __restrict__ partial, int chunks, long long cols,
                     uint16_t* __restrict__ out) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ float red[8][33];
  const long long s = blockIdx.y;
  const float t = reduce_rows_fixed(partial + s * chunks * cols, chunks, cols, cols, red);
  const long long c = (long long)blockIdx.x * 32 + (threadIdx.x & 31);
  if ((threadIdx.x >> 5) != 0 || c >= cols) return;
  __nv_bfloat16 v = __float2bfloat16_rn(t);
  out[s * cols + c] = *reinterpret_cast<uint16_t*>(&v);
}

int colsum_chunks(long long rows, long long cols, long long S) {
  const long long colblocks = (cols + 2047) / 2048;
  long long chunks = (4LL * sm_count()) / (colblocks * S);
  if (chunks < 1) chunks = 1;
  if (chunks > rows) chunks = rows;
  if (chunks > 1024) chunks = 1024;
  return (int)(chunks < 1 ? 1 : chunks);
}

}  // namespace

int layernorm_bwd_blocks(long long rows) {
  long long b = 2LL * sm_count();
  if (b > rows) b = rows;
  return (int)(b < 1 ? 1 : b);
}

size_t colsum_partial_floats(long long S, long long rows, long long cols) {
  if (rows < 1) rows = 1;
  return (size_t)S * (size_t)colsum_chunks(rows, cols, S) * (size_t)cols;
}

tp_status launch_colsum_stacked(const uint16_t* x, long long S, long long rows, long long cols,
                                uint16_t* out, float* partial, cudaStream_t stream, bool in_f16) {
  if (out == nullptr || cols == 0 || S == 0) return TP_OK;
  if (rows == 0) {
    return cuda_status(cudaMemsetAsync(out, 0, (size_t)(S * cols) * 2, stream));
  }
  const int chunks = colsum_chunks(rows, cols, S);
  const dim3 grid((unsigned)((cols + 2047) / 2048), (unsigned)chunks, (unsigned)S);
  {
    TraceScope ts(stream, TK_COLSUM);
    const int rpc = (int)((rows + chunks - 1) / chunks);
    if (in_f16)
      colsum_partial_kernel<true><<<grid, 256, 0, stream>>>(x, rows, cols, rpc, partial);
    else
      colsum_partial_kernel<false><<<grid, 256, 0, stream>>>(x, rows, cols, rpc, partial);
  }
  {
    TraceScope ts(stream, TK_COLSUM);
    const dim3 g2((unsigned)((cols + 31) / 32), (unsigned)S, 1);
    colsum_reduce_kernel<<<g2, 256, 0, stream>>>(partial, chunks, cols, out);
  }
  return cuda_status(cudaGetLastError());
}

tp_status launch_colsum_reduce(const float* partial, long long rows, long long cols, uint16_t* out,
                               cudaStream_t stream) {
  if (out == nullptr || cols == 0) return TP_OK;
  if (rows == 0) return cuda_status(cudaMemsetAsync(out, 0, (size_t)cols * 2, stream));
  TraceScope ts(stream, TK_COLSUM);
  const dim3 g2((unsigned)((cols + 31) / 32), 1, 1);
  launch_pdl(colsum_reduce_kernel, g2, dim3(256), 0, stream, (const float*)partial, (int)rows, cols,
             out);
  return cuda_status(cudaGetLastError());
}

template <bool F16OUT>
tp_status ln_fwd_dispatch(const uint16_t* x, const uint16_t* g, const uint16_t* b, long long rows,
                          int D, float eps, uint16_t* y, float* mean, float* rstd,
                          cudaStream_t stream) {
  long long nblk = (rows + 7) / 8;
  if (nblk > 2LL * sm_count()) nblk = 2LL * sm_count();
  const unsigned grid = (unsigned)nblk;
  const int per_lane = (D / 8 + 31) / 32;
  unsigned int* err = error_word();
  TraceScope ts(stream, TK_LN_FWD);
  if (per_lane <= 1)
    launch_pdl(ln_fwd_kernel<1, F16OUT>, dim3(grid), dim3(256), 0, stream, x, g, b, rows, D, eps, y,
               mean, rstd, err);
  else if (per_lane <= 2)
    launch_pdl(ln_fwd_kernel<2, F16OUT>, dim3(grid), dim3(256), 0, stream, x, g, b, rows, D, eps, y,
               mean, rstd, err);
  else if (per_lane <= 4)
    launch_pdl(ln_fwd_kernel<4, F16OUT>, dim3(grid), dim3(256), 0, stream, x, g, b, rows, D, eps, y,
               mean, rstd, err);
  else if (per_lane <= 8)
    launch_pdl(ln_fwd_kernel<8, F16OUT>, dim3(grid), dim3(256), 0, stream, x, g, b, rows, D, eps, y,
               mean, rstd, err);
  else if (per_lane <= 16)
    launch_pdl(ln_fwd_kernel<16, F16OUT>, dim3(grid), dim3(256), 0, stream, x, g, b, rows, D, eps, y,
               mean, rstd, err);
  else if (per_lane <= 32)
    launch_pdl(ln_fwd_kernel<32, F16OUT>, dim3(grid), dim3(256), 0, stream, x, g, b, rows, D, eps, y,
               mean, rstd, err);
  else
    return TP_ERR_UNSUPPORTED;
  return cuda_status(cudaGetLastError());
}

tp_status launch_layernorm_fwd(const uint16_t* x, const uint16_t* g, const uint16_t* b,
                               long long rows, int D, float eps, uint16_t* y, float* mean,
                               float* rstd, cudaStream_t stream, bool out_f16) {
  if (rows == 0) return TP_OK;
  if (out_f16) return ln_fwd_dispatch<true>(x, g, b, rows, D, eps, y, mean, rstd, stream);
  return ln_fwd_dispatch<false>(x, g, b, rows, D, eps, y, mean, rstd, stream);
}

size_t layernorm_bwd_partial_floats(long long rows, int D, int nk) {
  return (size_t)layernorm_bwd_blocks(rows < 1 ? 1 : rows) * (size_t)nk * (size_t)D;
}

namespace {
template <int CH, bool DY32>
void ln_bwd_kernel_launch(bool rsum, int nb, const void* dy, const uint16_t* x, const uint16_t* g,
                          const float* mean, const float* rstd, const uint16_t* dres,
                          long long rows, int D, int rpb, uint16_t* dx, float* partial,
                          float* dx32, cudaStream_t stream) {
  if (rsum)
    launch_pdl(ln_bwd_kernel<CH, DY32, true>, dim3(nb), dim3(LNB_THREADS), 0, stream, dy, x, g, mean,
               rstd, dres, rows, D, rpb, dx, partial, dx32);
  else
    launch_pdl(ln_bwd_kernel<CH, DY32, false>, dim3(nb), dim3(LNB_THREADS), 0, stream, dy, x, g,
               mean, rstd, dres, rows, D, rpb, dx, partial, dx32);
}

// dr (may be NULL; needs dres): column sums of dres, from a third partial row.
template <bool DY32>
tp_status ln_bwd_launch(const void* dy, const uint16_t* x, const uint16_t* g, const float* mean,
                        const float* rstd, const uint16_t* dres, long long rows, int D,
                        uint16_t* dx, float* dx32, uint16_t* dg, uint16_t* db, int nb,
                        float* partial, cudaStream_t stream, uint16_t* dr = nullptr) {
  if (dres == nullptr) dr = nullptr;
  if (rows == 0) {
    for (uint16_t* o : {dg, db, dr})
      if (o) cudaMemsetAsync(o, 0, (size_t)D * 2, stream);
    return cuda_status(cudaGetLastError());
  }
  if (nb < 1) return TP_ERR_INVALID_ARG;
  const int rpb = (int)((rows + nb - 1) / nb);
  const int per_thread = (D / 8 + LNB_THREADS - 1) / LNB_THREADS;
  const bool rsum = dr != nullptr;
  {
    TraceScope ts(stream, TK_LN_BWD);
    if (per_thread <= 1)
      ln_bwd_kernel_launch<1, DY32>(rsum, nb, dy, x, g, mean, rstd, dres, rows, D, rpb, dx,
                                    partial, dx32, stream);
    else if (per_thread <= 2)
      ln_bwd_kernel_launch<2, DY32>(rsum, nb, dy, x, g, mean, rstd, dres, rows, D, rpb, dx,
                                    partial, dx32, stream);
    else if (per_thread <= 4)
      ln_bwd_kernel_launch<4, DY32>(rsum, nb, dy, x, g, mean, rstd, dres, rows, D, rpb, dx,
                                    partial, dx32, stream);
    else
      return TP_ERR_UNSUPPORTED;
  }
  if (dg != nullptr || db != nullptr || dr != nullptr) {
    TraceScope ts(stream, TK_LN_PARAM);
    const int nk = rsum ? 3 : 2;
    launch_pdl(ln_param_reduce, dim3((nk * D + 31) / 32), dim3(256), 0, stream, (const float*)partial,
               nb, D, nk, dg, db, dr);
  }
  return cuda_status(cudaGetLastError());
}
}  // namespace

tp_status launch_layernorm_bwd(const uint16_t* dy, const uint16_t* x, const uint16_t* g,
                               const float* mean, const float* rstd, const uint16_t* dres,
                               long long rows, int D, uint16_t* dx, uint16_t* dg, uint16_t* db,
                               float* partial, cudaStream_t stream, float* dx32,
                               uint16_t* dres_sum) {
  return ln_bwd_launch<false>(dy, x, g, mean, rstd, dres, rows, D, dx, dx32, dg, db,
                              layernorm_bwd_blocks(rows < 1 ? 1 : rows), partial, stream,
                              dres_sum);
}

tp_status launch_layernorm_bwd_f32(const float* dy, const uint16_t* x, const uint16_t* g,
                                   const float* mean, const float* rstd, long long rows, int D,
                                   uint16_t* dx, float* dx32, uint16_t* dg, uint16_t* db,
                                   float* partial, cudaStream_t stream) {
  return ln_bwd_launch<true>(dy, x, g, mean, rstd, nullptr, rows, D, dx, dx32, dg, db,
                             layernorm_bwd_blocks(rows < 1 ? 1 : rows), partial, stream);
}

// LayerNorm backward with a caller-chosen number of row blocks `nb` (>= 1):
// `partial` must hold nb * 2 * D floats.  Used by the entry point whose
// scratch is a fixed-size static array.
tp_status launch_layernorm_bwd_blocks(const uint16_t* dy, const uint16_t* x, const uint16_t* g,
                                      const float* mean, const float* rstd, const uint16_t* dres,
                                      long long rows, int D, uint16_t* dx, uint16_t* dg,
                                      uint16_t* db, int nb, float* partial, cudaStream_t stream) {
  return ln_bwd_launch<false>(dy, x, g, mean, rstd, dres, rows, D, dx, nullptr, dg, db, nb,
                              partial, stream);
}

}  // namespace tp
