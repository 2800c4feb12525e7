// Persistent, warp-specialised tcgen05 GEMM for the sharded sublayer.
//
// C[m, n] = epilogue( sum_k A[m, k] * B[k, n] ), bf16 or fp16 operands (A and
// B of one type), fp32 accumulation in tensor memory, bf16, fp16 or fp32
// output.
//
// Tensor-parallel structure ("How transformer layers actually decompose",
// "The attention heads split"): the t shards of a column-parallel product
// appear as N shards (output [t][M][N/t]); the t partial products of a
// row-parallel product appear as K shards, walked one after the other into
// the SAME tensor-memory accumulator, so the cross-shard sum that the pages
// perform with an all-reduce happens in fp32 inside the MMA, in shard order
// 0..t-1, with a single rounding in the epilogue.  Weight-gradient products
// shard M or N the same way.
//
// Two kernels, both persistent with 320 threads (10 warps) per CTA:
//   gemm_pair_sm100 (M > 128): clusters of two CTAs on two SMs compute
//     256 x 256 tiles with tcgen05.mma.cta_group::2 (M = 256 split across the
//     pair).  Each CTA's producer stages its half of A and of B through a
//     6-stage TMA ring; the even CTA's single MMA thread issues 4 MMAs of
//     256 x 256 x 16 per 64-wide k-block into one of two 256-column TMEM
//     accumulators and commits stage releases to both CTAs.  One launch may
//     carry two independent products (their tiles one after the other in the
//     clusters' walk), so that two short products fill each other's partial
//     last round.
//   gemm_bf16_sm100 (M <= 128): one CTA per 128 x 256 tile, 4-stage ring,
//     4 MMAs of 128 x 256 x 16 per k-block.
// Roles in both: warp 0 TMA producer; warp 1 TMEM owner and MMA issuer (one
// thread); warps 2..9 epilogue, two per 32-lane quarter of tensor memory (a
// warp may only read its own quarter), each taking half of the tile's
// columns: tcgen05.ld, bias / GeLU (writing A and H) / GeLU-backward /
// residual (bf16 or fp32), then the stores.  The second accumulator lets the epilogue of tile i overlap the
// MMAs of tile i+1.  Tiles are visited in groups of 8 M-blocks per N sweep so
// that concurrently running tiles share A and B panels in L2.
// Every wait is bounded; a timeout records an error code and the kernel
// drains its own copies and MMAs, frees TMEM and returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "pdl.cuh"
#include "sm100_ptx.cuh"

namespace tp {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_BK = 64;        // one 128-byte swizzle row of bf16
constexpr int GEMM_STAGES = 4;
constexpr int GEMM_EPI_WARPS = 8;   // two per TMEM lane quarter, each draining half the columns
constexpr int GEMM_THREADS = 64 + 32 * GEMM_EPI_WARPS;
constexpr int GEMM_A_BYTES = GEMM_BM * GEMM_BK * 2;   // 16 KiB
constexpr int GEMM_B_BYTES = GEMM_BN * GEMM_BK * 2;   // 32 KiB
constexpr int GEMM_STAGE_BYTES = GEMM_A_BYTES + GEMM_B_BYTES;
constexpr int GEMM_SMEM_BYTES = GEMM_STAGES * GEMM_STAGE_BYTES + 1024 /*align*/ + 256 /*bars*/;
constexpr uint32_t GEMM_TMEM_COLS = 512;               // two 128x256 fp32 accumulators

enum EpiKind : int {
  EPI_LINEAR = 0,     // C = acc (+ bias[n]) (+ aux[m, n])
  EPI_BIAS_GELU = 1,  // C = acc (+ bias[n]);  C2 = GeLU(C)
  EPI_DGELU = 2,      // C = acc * GeLU'(aux[m, n])
};

enum ShardSrc : int { SHARD_NONE = 0, SHARD_K = 1, SHARD_MN = 2 };

// Error codes written to the library's device error word.
enum : unsigned int {
  ERR_GEMM_PRODUCER_WAIT = 0x101,
  ERR_GEMM_MMA_WAIT = 0x102,
  ERR_GEMM_EPI_WAIT = 0x103,
  ERR_GEMM_DRAIN_WAIT = 0x104,
  ERR_F16_RANGE = 0x301,          // a value stored as fp16 exceeded its range
};

struct GemmArgs {
  int m_shards, n_shards;          // output shards along M and along N
  int Mt, Nt;                      // rows / columns of one output shard
  int mb_per_shard, nb_per_shard;  // ceil(Mt / BM), ceil(Nt / BN)
  int k_shards, kb_per_shard;      // K walk: k_shards x ceil(Kt / BK) blocks
  int a_src, b_src;                // which index selects each operand's shard
  int num_tiles, group_m;
  int epi;
  // C element (ms, m, ns, n) lives at c + ms*c_ms + ns*c_ns + m*ldc + n; aux
  // (residual or saved pre-activation) and C2 share that layout; bias is
  // indexed by ns*Nt + n.
  __nv_bfloat16* c;
  __nv_bfloat16* c2;
  const __nv_bfloat16* aux;
  const __nv_bfloat16* bias;
  long long c_ms, c_ns, ldc;
  uint32_t idesc;                  // tcgen05 instruction descriptor (operand type, shape, majors)
  int a_il, b_il;                  // MN-major operand staged chunk-interleaved (see below)
  int out_f16;                     // C (and C2) stored as fp16 instead of bf16
  int out_f32;                     // C stored as fp32 (EPI_LINEAR only; `c` then points at floats)
  int aux_f32;                     // aux is an fp32 residual (EPI_LINEAR only)
  // Column sums of C (its fp32 values, before rounding), one partial row per
  // 32-row group: colpart[(m / 32) * colpart_ld + ns * Nt + n].  One M shard only.
  float* colpart;
  long long colpart_ld;
  unsigned int* err;
};

// tanh(u) from the hardware's tanh approximation: one special-function
// operation.  Its relative error (at most about 2^-11 by the PTX ISA's
// statement of the instruction) stays below the bf16 rounding of the stored
// GeLU and GeLU' results (2^-9); the GeLU products measured 1-2 % faster than
// with tanh built from the base-2 exponential and a reciprocal.
__device__ __forceinline__ float tanh_hw(float u) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(u));
  return t;
}

__device__ __forceinline__ float gelu_tanh_f(float a) {
  const float k0 = 0.7978845608028654f, k1 = 0.044715f;
  return 0.5f * a * (1.0f + tanh_hw(k0 * (a + k1 * a * a * a)));
}

__device__ __forceinline__ float gelu_tanh_grad_f(float a) {
  const float k0 = 0.7978845608028654f, k1 = 0.044715f;
  const float th = tanh_hw(k0 * (a + k1 * a * a * a));
  return 0.5f * (1.0f + th) + 0.5f * a * (1.0f - th * th) * k0 * (1.0f + 3.0f * k1 * a * a);
}

// Epilogue of 32 consecutive columns [n, n+32) of one output row: bias,
// residual (bf16 or fp32) or GeLU', store (bf16, fp16 or fp32), and GeLU into C2.  `base` is the
// row's element offset of C; columns past Nt are not touched.
__device__ __forceinline__ void epilogue_store32(const GemmArgs& p, float (&v)[32], int ns,
                                                 long long base, int n) {
  const int nvalid = min(32, p.Nt - n);   // a multiple of 8
  if (p.bias != nullptr && p.epi != EPI_DGELU) {
    const __nv_bfloat16* bp = p.bias + (long long)ns * p.Nt + n;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (g * 8 < nvalid) {
        const uint4 bv = *reinterpret_cast<const uint4*>(bp + g * 8);
        const uint32_t w[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          v[g * 8 + 2 * q] += bf16_lo(w[q]);
          v[g * 8 + 2 * q + 1] += bf16_hi(w[q]);
        }
      }
    }
  }
  if (p.aux != nullptr && p.aux_f32) {
    const float* xp = reinterpret_cast<const float*>(p.aux) + base + n;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (g * 8 < nvalid) {
        const float4 r0 = *reinterpret_cast<const float4*>(xp + g * 8);
        const float4 r1 = *reinterpret_cast<const float4*>(xp + g * 8 + 4);
        v[g * 8 + 0] += r0.x; v[g * 8 + 1] += r0.y; v[g * 8 + 2] += r0.z; v[g * 8 + 3] += r0.w;
        v[g * 8 + 4] += r1.x; v[g * 8 + 5] += r1.y; v[g * 8 + 6] += r1.z; v[g * 8 + 7] += r1.w;
      }
    }
  } else if (p.aux != nullptr) {
    const __nv_bfloat16* xp = p.aux + base + n;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (g * 8 < nvalid) {
        const uint4 av = *reinterpret_cast<const uint4*>(xp + g * 8);
        const uint32_t w[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float lo = bf16_lo(w[q]), hi = bf16_hi(w[q]);
          if (p.epi == EPI_DGELU) {
            v[g * 8 + 2 * q] *= gelu_tanh_grad_f(lo);
            v[g * 8 + 2 * q + 1] *= gelu_tanh_grad_f(hi);
          } else {
            v[g * 8 + 2 * q] += lo;
            v[g * 8 + 2 * q + 1] += hi;
          }
        }
      }
    }
  }
  __nv_bfloat16* cp = p.c + base + n;
  if (p.out_f32) {
    float* fp = reinterpret_cast<float*>(p.c) + base + n;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (g * 8 < nvalid) {
        *reinterpret_cast<float4*>(fp + g * 8) =
            make_float4(v[g * 8 + 0], v[g * 8 + 1], v[g * 8 + 2], v[g * 8 + 3]);
        *reinterpret_cast<float4*>(fp + g * 8 + 4) =
            make_float4(v[g * 8 + 4], v[g * 8 + 5], v[g * 8 + 6], v[g * 8 + 7]);
      }
    }
  } else if (p.out_f16) {
    bool over = false;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (g * 8 < nvalid) {
        uint4 o;
        o.x = pack_f16x2(v[g * 8 + 0], v[g * 8 + 1]);
        o.y = pack_f16x2(v[g * 8 + 2], v[g * 8 + 3]);
        o.z = pack_f16x2(v[g * 8 + 4], v[g * 8 + 5]);
        o.w = pack_f16x2(v[g * 8 + 6], v[g * 8 + 7]);
        *reinterpret_cast<uint4*>(cp + g * 8) = o;
#pragma unroll
        for (int e = 0; e < 8; ++e) over |= fabsf(v[g * 8 + e]) > 65504.0f;
      }
    }
    if (over && p.err) atomicCAS(p.err, 0u, ERR_F16_RANGE);
  } else {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (g * 8 < nvalid) {
        uint4 o;
        o.x = pack_bf16x2(v[g * 8 + 0], v[g * 8 + 1]);
        o.y = pack_bf16x2(v[g * 8 + 2], v[g * 8 + 3]);
        o.z = pack_bf16x2(v[g * 8 + 4], v[g * 8 + 5]);
        o.w = pack_bf16x2(v[g * 8 + 6], v[g * 8 + 7]);
        *reinterpret_cast<uint4*>(cp + g * 8) = o;
      }
    }
  }
  if (p.epi == EPI_BIAS_GELU) {
    __nv_bfloat16* hp = p.c2 + base + n;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (g * 8 < nvalid) {
        uint4 o;
        o.x = pack_bf16x2(gelu_tanh_f(v[g * 8 + 0]), gelu_tanh_f(v[g * 8 + 1]));
        o.y = pack_bf16x2(gelu_tanh_f(v[g * 8 + 2]), gelu_tanh_f(v[g * 8 + 3]));
        o.z = pack_bf16x2(gelu_tanh_f(v[g * 8 + 4]), gelu_tanh_f(v[g * 8 + 5]));
        o.w = pack_bf16x2(gelu_tanh_f(v[g * 8 + 6]), gelu_tanh_f(v[g * 8 + 7]));
        *reinterpret_cast<uint4*>(hp + g * 8) = o;
      }
    }
  }
}

// Sum over the warp's 32 lanes of each of the 32 columns in v: a transposing
// butterfly (at each of 5 stages a lane keeps one half of its columns, sends
// the other half to its partner and adds what it receives), after which lane
// l holds the sum of column l.  The order of the additions is fixed.
__device__ __forceinline__ float warp_colsum32(float (&v)[32]) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (threadIdx.x & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

// One 32-column chunk of an epilogue warp: the epilogue for rows inside the
// tensor, then (when asked) the warp's column sums.  `group` is the 32-row
// group of the warp's rows; rows past Mt contribute zero, and a group wholly
// past Mt (the tail of the last tile) writes nothing: the partial buffer holds
// ceil(Mt / 32) rows.
__device__ __forceinline__ void epilogue_chunk(const GemmArgs& p, const uint32_t (&r)[32], int ns,
                                               long long base, int n, bool row_ok, int group) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = row_ok ? __uint_as_float(r[i]) : 0.f;
  if (row_ok) epilogue_store32(p, v, ns, base, n);
  if (p.colpart != nullptr) {
    const float s = warp_colsum32(v);
    const int col = n + (int)(threadIdx.x & 31);
    if (col < p.Nt && group * 32 < p.Mt)
      p.colpart[(long long)group * p.colpart_ld + (long long)ns * p.Nt + col] = s;
  }
}

// Shared-memory descriptor of an MN-major operand tile of `chunks` 64-wide
// M/N chunks at K step kk (16 rows of K).  Two staging layouts:
//   interleaved (il): for each group of 8 K rows, the chunks' 1 KiB swizzle
//     atoms sit side by side (the canonical order: LBO = 1 KiB between chunks,
//     SBO = chunks KiB between 8-row K groups); one 5-D TMA box fills it;
//   chunk-major: each chunk holds all 64 K rows (8 KiB); LBO = 8 KiB,
//     SBO = 1 KiB; one 2-D box per chunk.
__device__ __forceinline__ uint64_t mn_desc(uint32_t base, int chunks, int kk, bool il) {
  return il ? smem_desc_sw128(base + kk * 2 * chunks * 1024, 1024, chunks * 1024)
            : smem_desc_sw128(base + kk * 2048, 8192, 1024);
}

struct TileCoord {
  int ms, m0, ns, n0;
};

__device__ __forceinline__ TileCoord gemm_tile(const GemmArgs& p, int tile) {
  const int mbt = p.m_shards * p.mb_per_shard;
  const int nbt = p.n_shards * p.nb_per_shard;
  const int per_group = p.group_m * nbt;
  const int g = tile / per_group;
  const int first = g * p.group_m;
  const int gsize = min(mbt - first, p.group_m);
  const int r = tile - g * per_group;
  const int mb = first + r % gsize;
  const int nb = r / gsize;
  TileCoord tc;
  tc.ms = mb / p.mb_per_shard;
  tc.m0 = (mb - tc.ms * p.mb_per_shard) * GEMM_BM;
  tc.ns = nb / p.nb_per_shard;
  tc.n0 = (nb - tc.ns * p.nb_per_shard) * GEMM_BN;
  return tc;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > 2000000000ull) return false;
  }
}

__device__ __forceinline__ void record_error(unsigned int* err, volatile int* abort_flag,
                                             unsigned int code) {
  *abort_flag = 1;
  if (err) atomicCAS(err, 0u, code);
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
gemm_bf16_sm100(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + GEMM_STAGES * GEMM_STAGE_BYTES);
  uint64_t* full = bars;                        // [STAGES]
  uint64_t* empty = bars + GEMM_STAGES;         // [STAGES]
  uint64_t* tfull = bars + 2 * GEMM_STAGES;     // [2]
  uint64_t* tempty = tfull + 2;                 // [2]
  uint64_t* drain = tempty + 2;                 // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < GEMM_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 32 * GEMM_EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, GEMM_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = p.k_shards * p.kb_per_shard;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        const TileCoord tc = gemm_tile(p, tile);
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % GEMM_STAGES;
          const uint32_t round = it / GEMM_STAGES;
          if (!wait_or_abort(&empty[s], (round & 1) ^ 1, abort_flag)) {
            record_error(p.err, abort_flag, ERR_GEMM_PRODUCER_WAIT);
            ok = false;
            break;
          }
          const int ks = kb / p.kb_per_shard;
          const int k0 = (kb - ks * p.kb_per_shard) * GEMM_BK;
          const int a_s = p.a_src == SHARD_K ? ks : (p.a_src == SHARD_MN ? tc.ms : 0);
          const int b_s = p.b_src == SHARD_K ? ks : (p.b_src == SHARD_MN ? tc.ns : 0);
          uint8_t* sa = smem + s * GEMM_STAGE_BYTES;
          uint8_t* sb = sa + GEMM_A_BYTES;
          mbar_arrive_expect_tx(&full[s], GEMM_STAGE_BYTES);
          if (A_MN && p.a_il) {
            tma_load_5d(sa, &tmA, &full[s], 0, 0, tc.m0 / 64, k0 / 8, a_s);
          } else if (A_MN) {
#pragma unroll
            for (int j = 0; j < GEMM_BM / 64; ++j)
              tma_load_3d(sa + j * 8192, &tmA, &full[s], tc.m0 + 64 * j, k0, a_s);
          } else {
            tma_load_3d(sa, &tmA, &full[s], k0, tc.m0, a_s);
          }
          if (B_MN && p.b_il) {
            tma_load_5d(sb, &tmB, &full[s], 0, 0, tc.n0 / 64, k0 / 8, b_s);
          } else if (B_MN) {
#pragma unroll
            for (int j = 0; j < GEMM_BN / 64; ++j)
              tma_load_3d(sb + j * 8192, &tmB, &full[s], tc.n0 + 64 * j, k0, b_s);
          } else {
            tma_load_3d(sb, &tmB, &full[s], k0, tc.n0, b_s);
          }
        }
      }
      // Let every copy this thread issued land before the CTA can exit.
      const int issued = it;
      for (int j = 0; j < GEMM_STAGES && j < issued; ++j) {
        const int i = issued - 1 - j;
        mbar_wait(&full[i % GEMM_STAGES], (i / GEMM_STAGES) & 1, 200000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = p.idesc;
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tcount) {
        const int acc = tcount & 1;
        const uint32_t use = tcount >> 1;
        if (!wait_or_abort(&tempty[acc], (use & 1) ^ 1, abort_flag)) {
          record_error(p.err, abort_flag, ERR_GEMM_MMA_WAIT);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * GEMM_BN;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % GEMM_STAGES;
          const uint32_t round = it / GEMM_STAGES;
          if (!wait_or_abort(&full[s], round & 1, abort_flag)) {
            record_error(p.err, abort_flag, ERR_GEMM_MMA_WAIT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * GEMM_STAGE_BYTES);
          const uint32_t sb = sa + GEMM_A_BYTES;
#pragma unroll
          for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
            const uint64_t ad = A_MN ? mn_desc(sa, GEMM_BM / 64, kk, p.a_il)
                                     : smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? mn_desc(sb, GEMM_BN / 64, kk, p.b_il)
                                     : smem_desc_sw128(sb + kk * 32, 16, 1024);
            tc_mma_f16(d_tmem, ad, bd, idesc, (kb | kk) != 0);
          }
          tc_commit(&empty[s]);   // frees the stage once these MMAs have read it
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);   // accumulator ready for the epilogue
      }
      // Drain: every MMA issued above has completed before TMEM is freed.
      tc_commit(drain);
      if (!mbar_wait(drain, 0, 200000000ull)) record_error(p.err, abort_flag, ERR_GEMM_DRAIN_WAIT);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;                 // TMEM lane quarter this warp may access
    const int row = quad * 32 + lane;          // row within the tile
    constexpr int CPW = GEMM_BN / 32 / (GEMM_EPI_WARPS / 4);   // 32-column chunks per warp
    const int c0 = ((warp - 2) / 4) * CPW;
    int tcount = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
      const TileCoord tc = gemm_tile(p, tile);
      const int acc = tcount & 1;
      const uint32_t use = tcount >> 1;
      // Warp-uniform outcome: the tcgen05.ld below is a warp-collective instruction.
      if (!__all_sync(0xffffffffu, wait_or_abort(&tfull[acc], use & 1, abort_flag))) {
        record_error(p.err, abort_flag, ERR_GEMM_EPI_WAIT);
        break;
      }
      tc_fence_after();
      const int m = tc.m0 + row;
      const bool row_ok = m < p.Mt;
      const long long base = tc.ms * p.c_ms + tc.ns * p.c_ns + (long long)m * p.ldc;
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * GEMM_BN;
#pragma unroll 1
      for (int c = c0; c < c0 + CPW; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        tc_wait_ld();
        const int n = tc.n0 + c * 32;
        if (n >= p.Nt) continue;   // the same for every lane of the warp
        epilogue_chunk(p, r, tc.ns, base, n, row_ok, (tc.m0 + quad * 32) / 32);
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, GEMM_TMEM_COLS);
  }
}

// =====================================================================================
// CTA-pair variant (tcgen05 cta_group::2): a cluster of two CTAs computes one
// 256 x 256 tile.  Each CTA streams its own 128 rows of A and its own half
// (128 columns) of B; one thread of the even CTA issues 256 x 256 x 16 MMAs
// that read A and B from both CTAs' shared memory and write each CTA's 128
// rows into that CTA's tensor memory.  Per SM this halves the B tile it has
// to fetch and stage compared with the single-CTA kernel.
// =====================================================================================
constexpr int GP_BM = 256;                 // rows per pair tile (128 per CTA)
constexpr int GP_BN = 256;                 // columns per pair tile (128 of B per CTA)
constexpr int GP_STAGES = 6;
constexpr int GP_A_BYTES = 128 * GEMM_BK * 2;   // 16 KiB per CTA
constexpr int GP_B_BYTES = 128 * GEMM_BK * 2;   // 16 KiB per CTA
constexpr int GP_STAGE_BYTES = GP_A_BYTES + GP_B_BYTES;
constexpr int GP_SMEM_BYTES = GP_STAGES * GP_STAGE_BYTES + 1024 + 256;

enum : unsigned int {
  ERR_GEMMP_PRODUCER_WAIT = 0x111,
  ERR_GEMMP_MMA_WAIT = 0x112,
  ERR_GEMMP_EPI_WAIT = 0x113,
};

__device__ __forceinline__ TileCoord gemm_pair_tile(const GemmArgs& p, int tile) {
  const int mbt = p.m_shards * p.mb_per_shard;
  const int nbt = p.n_shards * p.nb_per_shard;
  const int per_group = p.group_m * nbt;
  const int g = tile / per_group;
  const int first = g * p.group_m;
  const int gsize = min(mbt - first, p.group_m);
  const int r = tile - g * per_group;
  const int mb = first + r % gsize;
  const int nb = r / gsize;
  TileCoord tc;
  tc.ms = mb / p.mb_per_shard;
  tc.m0 = (mb - tc.ms * p.mb_per_shard) * GP_BM;
  tc.ns = nb / p.nb_per_shard;
  tc.n0 = (nb - tc.ns * p.nb_per_shard) * GP_BN;
  return tc;
}

// Two products in one launch: tiles 0 .. p.num_tiles-1 are product p (maps
// tmA, tmB), the next p2.num_tiles are product p2 (maps tmA2, tmB2; same
// operand majors and type).  One launch of two products whose tile counts
// leave partial last rounds of clusters fills those rounds with each other's
// tiles.  p2.num_tiles = 0 for a single product.
template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
gemm_pair_sm100(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ GemmArgs p, const __grid_constant__ CUtensorMap tmA2,
                const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ GemmArgs p2) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + GP_STAGES * GP_STAGE_BYTES);
  uint64_t* full = bars;                      // [STAGES], counted in the even CTA
  uint64_t* empty = bars + GP_STAGES;         // [STAGES], one per CTA
  uint64_t* tfull = bars + 2 * GP_STAGES;     // [2]
  uint64_t* tempty = tfull + 2;               // [2], counted in the even CTA
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < GP_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * GEMM_EPI_WARPS);   // one arrival per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (p2.num_tiles > 0) {
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB2);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, GEMM_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();                   // the peer's barriers exist before anyone signals them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int cid = (int)cluster_id_x(), ncl = (int)nclusters_x();
  const int ntiles = p.num_tiles + p2.num_tiles;
  grid_dep_wait();                  // operands and outputs: the previous kernels have completed
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      // One tile's k-blocks; called with the kernel parameter of its product
      // itself, so that every field is read from the parameter space.
      auto produce = [&](const GemmArgs& q, const CUtensorMap* ta, const CUtensorMap* tb,
                         int ltile) {
        const TileCoord tc = gemm_pair_tile(q, ltile);
        const int am = tc.m0 + (int)rank * 128;
        const int bn = tc.n0 + (int)rank * 128;
        const int num_kb = q.k_shards * q.kb_per_shard;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % GP_STAGES;
          const uint32_t round = it / GP_STAGES;
          if (!wait_or_abort(&empty[s], (round & 1) ^ 1, abort_flag)) {
            record_error(p.err, abort_flag, ERR_GEMMP_PRODUCER_WAIT);
            return false;
          }
          const int ks = kb / q.kb_per_shard;
          const int k0 = (kb - ks * q.kb_per_shard) * GEMM_BK;
          const int a_s = q.a_src == SHARD_K ? ks : (q.a_src == SHARD_MN ? tc.ms : 0);
          const int b_s = q.b_src == SHARD_K ? ks : (q.b_src == SHARD_MN ? tc.ns : 0);
          uint8_t* sa = smem + s * GP_STAGE_BYTES;
          uint8_t* sb = sa + GP_A_BYTES;
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * GP_STAGE_BYTES);
          if (A_MN && q.a_il) {
            tma_load_5d_pair(sa, ta, &full[s], 0, 0, am / 64, k0 / 8, a_s);
          } else if (A_MN) {
            tma_load_3d_pair(sa, ta, &full[s], am, k0, a_s);
            tma_load_3d_pair(sa + 8192, ta, &full[s], am + 64, k0, a_s);
          } else {
            tma_load_3d_pair(sa, ta, &full[s], k0, am, a_s);
          }
          if (B_MN && q.b_il) {
            tma_load_5d_pair(sb, tb, &full[s], 0, 0, bn / 64, k0 / 8, b_s);
          } else if (B_MN) {
            tma_load_3d_pair(sb, tb, &full[s], bn, k0, b_s);
            tma_load_3d_pair(sb + 8192, tb, &full[s], bn + 64, k0, b_s);
          } else {
            tma_load_3d_pair(sb, tb, &full[s], k0, bn, b_s);
          }
        }
        return true;
      };
      for (int tile = cid; tile < ntiles && ok; tile += ncl)
        ok = tile < p.num_tiles ? produce(p, &tmA, &tmB, tile)
                                : produce(p2, &tmA2, &tmB2, tile - p.num_tiles);
      if (leader) {
        const int issued = it;
        for (int j = 0; j < GP_STAGES && j < issued; ++j) {
          const int i = issued - 1 - j;
          mbar_wait(&full[i % GP_STAGES], (i / GP_STAGES) & 1, 200000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      if (leader) {
        int it = 0, tcount = 0;
        bool ok = true;
        for (int tile = cid; tile < ntiles && ok; tile += ncl, ++tcount) {
          const bool sec = tile >= p.num_tiles;
          const uint32_t idesc = sec ? p2.idesc : p.idesc;
          const int num_kb = sec ? p2.k_shards * p2.kb_per_shard : p.k_shards * p.kb_per_shard;
          const bool a_il = sec ? p2.a_il : p.a_il, b_il = sec ? p2.b_il : p.b_il;
          const int acc = tcount & 1;
          const uint32_t use = tcount >> 1;
          if (!wait_or_abort(&tempty[acc], (use & 1) ^ 1, abort_flag)) {
            record_error(p.err, abort_flag, ERR_GEMMP_MMA_WAIT);
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * GP_BN;
          for (int kb = 0; kb < num_kb; ++kb, ++it) {
            const int s = it % GP_STAGES;
            const uint32_t round = it / GP_STAGES;
            if (!wait_or_abort(&full[s], round & 1, abort_flag)) {
              record_error(p.err, abort_flag, ERR_GEMMP_MMA_WAIT);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + s * GP_STAGE_BYTES);
            const uint32_t sb = sa + GP_A_BYTES;
#pragma unroll
            for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
              const uint64_t ad = A_MN ? mn_desc(sa, 2, kk, a_il)
                                       : smem_desc_sw128(sa + kk * 32, 16, 1024);
              const uint64_t bd = B_MN ? mn_desc(sb, 2, kk, b_il)
                                       : smem_desc_sw128(sb + kk * 32, 16, 1024);
              tc_mma_f16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0);
            }
            tc_commit_pair(&empty[s], 0x3);   // frees stage s in both CTAs
          }
          if (!ok) break;
          tc_commit_pair(&tfull[acc], 0x3);   // both CTAs' accumulators ready
        }
        tc_commit_pair(drain, 0x3);
      }
      if (!mbar_wait(drain, 0, 200000000ull)) record_error(p.err, abort_flag, ERR_GEMM_DRAIN_WAIT);
    }
  } else {
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    constexpr int CPW = GP_BN / 32 / (GEMM_EPI_WARPS / 4);     // 32-column chunks per warp
    const int c0 = ((warp - 2) / 4) * CPW;
    const uint32_t tempty_leader0 = map_to_rank(&tempty[0], 0);
    int tcount = 0;
    // One tile's epilogue, called like the producer's with its product's
    // kernel parameter itself.
    auto drain_tile = [&](const GemmArgs& q, int ltile, int acc) {
      const TileCoord tc = gemm_pair_tile(q, ltile);
      const int m = tc.m0 + (int)rank * 128 + row;
      const bool row_ok = m < q.Mt;
      const long long base = tc.ms * q.c_ms + tc.ns * q.c_ns + (long long)m * q.ldc;
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * GP_BN;
#pragma unroll 1
      for (int c = c0; c < c0 + CPW; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        tc_wait_ld();
        const int n = tc.n0 + c * 32;
        if (n >= q.Nt) continue;   // the same for every lane of the warp
        epilogue_chunk(q, r, tc.ns, base, n, row_ok, (tc.m0 + (int)rank * 128 + quad * 32) / 32);
      }
    };
    for (int tile = cid; tile < ntiles; tile += ncl, ++tcount) {
      const int acc = tcount & 1;
      const uint32_t use = tcount >> 1;
      if (!__all_sync(0xffffffffu, wait_or_abort(&tfull[acc], use & 1, abort_flag))) {
        record_error(p.err, abort_flag, ERR_GEMMP_EPI_WAIT);
        break;
      }
      tc_fence_after();
      if (tile < p.num_tiles) drain_tile(p, tile, acc);
      else drain_tile(p2, tile - p.num_tiles, acc);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + acc * 8);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();                   // no CTA leaves while its pair may still read its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, GEMM_TMEM_COLS);
  }
}

}  // namespace tp
