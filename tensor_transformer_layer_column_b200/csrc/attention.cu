// Per-head causal attention on tcgen05, over the shard-packed projections.
//
// "The attention heads split": shard i owns heads i*H/t .. (i+1)*H/t-1 and
// runs full attention for them with no communication.  The projections arrive
// as qkv [t][T][3Dt] (the column-parallel GEMM's output, fp16): local head j
// of shard i has q at columns j*dh, k at Dt + j*dh, v at 2Dt + j*dh of rows
// b*S + s.  One launch covers every head of every shard.
//
// Operand precision: q, k, v, P, dO and dS are fp16 (10-bit mantissa) rather
// than bf16.  Over long causal rows the softmax amplifies the storage
// rounding of q and k (and of the LayerNorm output they come from); with
// bf16 storage that alone puts the relative L2 error of O and of dWout near
// 6e-3 at S = 2048, with fp16 near 2e-3.  The tensor-core rate is the same.
//
// Forward (per pair of 128-query tiles, head, batch; 64-key blocks):
//   S = q k^T (tcgen05, fp32 in TMEM), online softmax in fp32 by one thread per
//   query row (base-2 exponent, scores pre-scaled by log2(e)/sqrt(dh)), P
//   rounded to fp16 into tensor memory, O += P v (tcgen05 with P as the
//   A operand read from tensor memory, fp32 in TMEM, rescaled lazily).  The
//   two tiles alternate on the tensor core.
//   Writes O [t][T][Dt] (bf16) and the log-sum-exp [B][H][S] (fp32).
// Backward (P recomputed from the log-sum-exp; no atomics, deterministic;
// dO in and dqkv out are fp16):
//   prep:   Dv = rowsum(dO * O), lse2 = lse * log2(e)
//   dK/dV:  per 128-key block, walk 64-query blocks:  S^T = k q^T, dP^T = v dO^T,
//           P^T, dS^T = P^T * (dP^T - Dv) by one thread per key row,
//           dV += P^T dO, dK += dS^T q; also stores dS^T (fp16) when the
//           array fits under the limit attn_set_dst_limit sets
//   dQ:     per 256-query block, walk 64-key blocks: dQ += dS k, dS read
//           back from that array; above the limit a dQ kernel over 128-query
//           blocks recomputes S = q k^T, dP = dO v^T, dS = P * (dP - Dv)
//           instead
//   dK/dV and the recomputing dQ are persistent: one CTA per SM walks its
//   work items (snake order, longest first) with the pipelines carried from
//   item to item and four epilogue warps writing an item's dK/dV or dQ while
//   the next one starts.
// P, P^T, dS^T and dS go from registers to tensor memory (fp16) and are the
// A operands of the products that consume them, read from there: shared
// memory, whose bandwidth the score products already use up, carries only
// the TMA tiles and the B operands.
// Every wait is bounded (about 2 s); a timeout records an error code and the
// kernel drains its copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace tp {

namespace {

enum : unsigned int {
  ERR_ATTN_FWD_WAIT = 0x201,
  ERR_ATTN_DKDV_WAIT = 0x202,
  ERR_ATTN_DQ_WAIT = 0x203,
};

// Compile-time flag for generic lambdas: one code path with the causal
// select, one without, chosen per block.
template <bool B>
struct BoolTag {
  static constexpr bool value = B;
};

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct AttnArgs {
  int B, S, H, Ht, Dt, t;
  int S_pad;            // bwd: row length of lse2 / dvec per (batch, head), a multiple of 128
  int causal;
  long long T;
  float scale_log2;     // log2(e) / sqrt(dh)
  float inv_sqrt_dh;
  uint16_t* out;        // fwd: o_save [t][T][Dt]; bwd: dqkv [t][T][3Dt]
  float* lse;           // fwd: lse [B][H][S]
  const float* lse2;    // bwd: lse * log2(e), [B][H][S_pad]; +inf past S
  const float* dvec;    // bwd: rowsum(dO * O), [B][H][S_pad]; 0 past S
  // bwd (may be null): column sums of dqkv for its bias gradient, one fp32
  // partial row per 32 rows of one batch element: colpart[(b * G + s / 32) *
  // (t * 3Dt) + shard * 3Dt + column], G = ceil(S / 32).
  float* colpart;
  // bwd (may be null): dS^T in fp16, written by the dK/dV kernel for the dQ
  // kernel that reads it (attn_bwd_dq_ds_kernel), in 4 KiB pieces of 32 keys x
  // 64 queries: piece (bh, j, i) holds keys 32i .. 32i+31 and queries 64j ..
  // 64j+63 of head bh = b*H + h at element ((bh * S_pad/64 + j) * S_pad/32 + i)
  // * 2048, one 128-byte row per key with its 16-byte chunks in the 128-byte
  // swizzle (chunk c of row r at position c ^ (r % 8)) -- the image of an
  // MN-major tensor-core operand tile, copied as is both ways.
  uint16_t* dst;
  unsigned int* err;
};

// Sum over the warp's 32 lanes of each of the 32 columns in v (a transposing
// butterfly; lane l ends with column l).  The order of additions is fixed.
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

// Writes the warp's column sums of 32 columns starting at shard column `col0`
// (rows of the warp: s0 .. s0 + 31 of batch element b; rows past S hold 0).
__device__ __forceinline__ void colpart_store(const AttnArgs& p, float (&v)[32], int b, int s0,
                                              int shard, int col0) {
  const float sum = warp_colsum32(v);
  const long long w3 = 3LL * p.Dt;
  const long long slot = (long long)b * ((p.S + 31) / 32) + s0 / 32;
  if (s0 < p.S)
    p.colpart[slot * (p.t * w3) + shard * w3 + col0 + (threadIdx.x & 31)] = sum;
}

struct Ctl {
  volatile int* abort_flag;
  unsigned int* err;
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Ctl& c,
                                         unsigned int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*c.abort_flag || globaltimer_ns() - t0 > 2000000000ull) {
      *c.abort_flag = 1;
      if (c.err) atomicCAS(c.err, 0u, code);
      return false;
    }
  }
}

// Item of a persistent CTA's k-th round: rounds alternate direction over the
// CTAs (snake order: CTA c takes item G*k + c in even rounds and
// G*k + G-1-c in odd ones), so that with items sorted longest first every CTA
// gets a near-equal share of the work (for the c5 dK/dV items, 1.2 % above the
// mean at most, against 6.3 % for round robin).  >= nitems: no item in this
// round (only in the last one).
__device__ __forceinline__ int snake_item(int k) {
  const int G = (int)gridDim.x, c = (int)blockIdx.x;
  return G * k + ((k & 1) ? G - 1 - c : c);
}

__device__ __forceinline__ uint4 pack8_f16(const float* v) {
  uint4 o;
  o.x = pack_f16x2(v[0], v[1]);
  o.y = pack_f16x2(v[2], v[3]);
  o.z = pack_f16x2(v[4], v[5]);
  o.w = pack_f16x2(v[6], v[7]);
  return o;
}

__device__ __forceinline__ uint4 pack8_bf16(const float* v) {
  uint4 o;
  o.x = pack_bf16x2(v[0], v[1]);
  o.y = pack_bf16x2(v[2], v[3]);
  o.z = pack_bf16x2(v[4], v[5]);
  o.w = pack_bf16x2(v[6], v[7]);
  return o;
}

// K-major operand descriptor for a tile of R rows x (64*chunks) columns, at K step kk (16 cols).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int R, int kk) {
  return smem_desc_sw128(base + (kk >> 2) * R * 128 + (kk & 3) * 32, 16, 1024);
}

// MN-major operand descriptor: tile rows are the K index (R rows), columns the
// M/N index in 64-wide chunks of R*128 bytes; K step kk covers rows 16kk..16kk+15.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, int R, int kk) {
  return smem_desc_sw128(base + kk * 2048, R * 128, 1024);
}

// =====================================================================================
// Forward
// =====================================================================================
// Two 128-query tiles per CTA take turns on the tensor core: while one tile's
// softmax warpgroup works on its scores, the other tile's products run.  Keys
// come in 64-wide blocks through a 4-stage ring; each tile has its own S (64
// TMEM columns), P (32 columns of fp16 pairs) and O (dh columns).  O is rescaled lazily: only when a row's
// running max grows by more than 2^8 (log2 units), so P = 2^(s - m_used) stays
// below 256 (exact in fp16) and the final O / l is unchanged.
template <int DH>
struct FwdCfg {
  static constexpr int BM = 128, BN = 64, CH = DH / 64, STAGES = 4;
  static constexpr int THREADS = 352;                   // producer, S issuer, 2 x 4 softmax warps, P V issuer
  static constexpr int Q_BYTES = BM * DH * 2;           // one query tile
  static constexpr int KV_BYTES = BN * DH * 2;          // K or V of one stage
  static constexpr int OFF_Q = 0;                       // tile i at +i*Q
  static constexpr int OFF_KV = 2 * Q_BYTES;            // stage s: K at +2s*KV, V at +(2s+1)*KV
  static constexpr int OFF_BAR = OFF_KV + STAGES * 2 * KV_BYTES;
  static constexpr int RAW = OFF_BAR + 256 + 1024;
  static constexpr int SMEM = RAW > 120 * 1024 ? RAW : 120 * 1024;   // one CTA per SM (512 TMEM columns)
};

static_assert(FwdCfg<128>::SMEM <= 227 * 1024, "forward tile exceeds shared memory");

constexpr float kLazyRescaleLog2 = 8.0f;

// Work item of a CTA in a (length index, head, batch) grid, longest first.
// Blocks start in linear order (x fastest); read as one index, the length
// index varies slowest, so every CTA of the first length index (the longest
// causal items) starts before any of the next, and the CTAs that start last,
// filling the tail of the launch, are the shortest.
struct AttnItem {
  int x, h, b;
};
__device__ __forceinline__ AttnItem attn_item() {
  const unsigned hb = gridDim.y * gridDim.z;
  const unsigned lin = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  AttnItem it;
  it.x = (int)(lin / hb);
  const unsigned r = lin - (unsigned)it.x * hb;
  it.h = (int)(r % gridDim.y);
  it.b = (int)(r / gridDim.y);
  return it;
}

template <int DH>
__global__ void __launch_bounds__(352, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q128,
                const __grid_constant__ CUtensorMap tm_kv64, const AttnArgs p) {
  using C = FwdCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;     // [STAGES <= 4]
  uint64_t* kv_empty = bars + 5;    // [STAGES]
  uint64_t* s_full = bars + 9;      // [2] per tile
  uint64_t* s_free = bars + 11;     // [2]
  uint64_t* p_full = bars + 13;     // [2]
  uint64_t* pv_done = bars + 15;    // [2]
  uint64_t* drain = bars + 17;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (p.S + 2 * C::BM - 1) / (2 * C::BM);
  const AttnItem item = attn_item();
  const int qb = p.causal ? nqb - 1 - item.x : item.x;
  const int h = item.h, b = item.b;
  const int shard = h / p.Ht, hl = h - shard * p.Ht;
  const int q0 = qb * 2 * C::BM;
  const int nkb = (p.S + C::BN - 1) / C::BN;
  int ntile[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int qs = q0 + i * C::BM;
    ntile[i] = qs >= p.S ? 0 : (p.causal ? min(nkb, (qs + C::BM) / C::BN) : nkb);
  }
  const int nkv = max(ntile[0], ntile[1]);
  const int colq = hl * DH, colk = p.Dt + hl * DH, colv = 2 * p.Dt + hl * DH;
  const Ctl ctl{abort_flag, p.err};

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q128);
    tma_prefetch_desc(&tm_kv64);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // TMEM columns: S of tile i at 64i, O of tile i at 128 + 128i, P of tile i at 384 + 32i.
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();   // inputs and outputs: the previous kernels have completed
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, 2 * C::Q_BYTES);
      for (int i = 0; i < 2; ++i)
        for (int c = 0; c < C::CH; ++c)
          tma_load_4d(smem + C::OFF_Q + i * C::Q_BYTES + c * C::BM * 128, &tm_q128, q_full,
                      colq + 64 * c, q0 + i * C::BM, b, shard);
      int j = 0;
      for (; j < nkv; ++j) {
        const int st = j % C::STAGES;
        const uint32_t u = j / C::STAGES;
        if (!wait_bar(&kv_empty[st], (u & 1) ^ 1, ctl, ERR_ATTN_FWD_WAIT)) break;
        uint8_t* sk = smem + C::OFF_KV + st * 2 * C::KV_BYTES;
        uint8_t* sv = sk + C::KV_BYTES;
        mbar_arrive_expect_tx(&kv_full[st], 2 * C::KV_BYTES);
        for (int c = 0; c < C::CH; ++c) {
          tma_load_4d(sk + c * C::BN * 128, &tm_kv64, &kv_full[st], colk + 64 * c, j * C::BN, b, shard);
          tma_load_4d(sv + c * C::BN * 128, &tm_kv64, &kv_full[st], colv + 64 * c, j * C::BN, b, shard);
        }
      }
      mbar_wait(q_full, 0, 200000000ull);
      for (int i = j - 1; i >= 0 && i >= j - C::STAGES; --i)
        mbar_wait(&kv_full[i % C::STAGES], (i / C::STAGES) & 1, 200000000ull);
    }
  } else if (warp == 1 || warp == 10) {
    // Two issuers, each blocking only on its own barriers: warp 1 issues the
    // scores S = q k^T of both tiles (block j+1 once the tile's softmax has
    // copied S of block j out of tensor memory), warp 10 the products P V
    // (once P is in tensor memory) and releases each K/V stage.  Neither
    // stream waits behind the other.
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_f32acc(128, C::BN, false, false, true);
      constexpr uint32_t id_pv = idesc_f32acc(128, DH, false, true, true);
      const uint32_t sq = smem_u32(smem + C::OFF_Q);
      auto kv_addr = [&](int j) { return smem_u32(smem + C::OFF_KV + (j % C::STAGES) * 2 * C::KV_BYTES); };
      bool ok = wait_bar(q_full, 0, ctl, ERR_ATTN_FWD_WAIT);
      if (warp == 1) {
        for (int j = 0; ok && j < nkv; ++j) {
          bool kv_in = false;   // block j has landed (waited for once)
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (ok && j < ntile[i]) {
              if (j > 0 && !(ok = wait_bar(&s_free[i], (j - 1) & 1, ctl, ERR_ATTN_FWD_WAIT))) break;
              if (!kv_in && !(ok = wait_bar(&kv_full[j % C::STAGES], (j / C::STAGES) & 1, ctl,
                                            ERR_ATTN_FWD_WAIT)))
                break;
              kv_in = true;
              tc_fence_after();
              const uint32_t sk = kv_addr(j);
#pragma unroll
              for (int kk = 0; kk < DH / 16; ++kk)
                tc_mma_f16(tmem + 64 * i, kmajor_desc(sq + i * C::Q_BYTES, C::BM, kk),
                           kmajor_desc(sk, C::BN, kk), id_s, kk > 0);
              tc_commit(&s_full[i]);
            }
          }
        }
      } else {
        for (int j = 0; ok && j < nkv; ++j) {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (ok && j < ntile[i]) {
              if (!(ok = wait_bar(&p_full[i], j & 1, ctl, ERR_ATTN_FWD_WAIT))) break;
              tc_fence_after();
              const uint32_t sv = kv_addr(j) + C::KV_BYTES;
#pragma unroll
              for (int kk = 0; kk < C::BN / 16; ++kk)   // 16 keys = 8 columns of P per step
                tc_mma_f16_ts(tmem + 128 + 128 * i, tmem + 384 + 32 * i + 8 * kk,
                              mnmajor_desc(sv, C::BN, kk), id_pv, (j | kk) != 0);
              tc_commit(&pv_done[i]);
            }
          }
          if (!ok) break;
          // The scores of block j completed before its softmax produced P, so
          // once these products complete nothing reads the stage any more.
          tc_commit(&kv_empty[j % C::STAGES]);
        }
        tc_commit(drain);
        mbar_wait(drain, 0, 200000000ull);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax warpgroups
    const int tile = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int qt = q0 + tile * C::BM;
    const int q = qt + r;
    const int n = ntile[tile];
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t t_s = tmem + 64 * tile + lane_off;
    const uint32_t t_o = tmem + 128 + 128 * tile + lane_off;
    const uint32_t t_p = tmem + 384 + 32 * tile + lane_off;
    float m_used = -1e30f, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      if (!__all_sync(0xffffffffu, wait_bar(&s_full[tile], j & 1, ctl, ERR_ATTN_FWD_WAIT))) { ok = false; break; }
      tc_fence_after();
      float s[C::BN];
      {
        uint32_t ra[32], rb[32];
        tmem_ld32(t_s, ra);
        tmem_ld32(t_s + 32, rb);
        tc_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          s[e] = __uint_as_float(ra[e]);
          s[32 + e] = __uint_as_float(rb[e]);
        }
      }
      tc_fence_before();
      mbar_arrive(&s_free[tile]);
      // Keys past the last visible one (after the query, or past S) are masked: a select
      // per element against a bound fixed once per block, taken only in blocks where
      // some row of the warp has a masked key (the causal diagonal, the sequence end).
      const int kmax = (p.causal ? min(q, p.S - 1) : p.S - 1) - j * C::BN;
      if (!__all_sync(0xffffffffu, kmax >= C::BN - 1)) {
#pragma unroll
        for (int c = 0; c < C::BN; ++c) s[c] = c > kmax ? -INFINITY : s[c];
      }
      // Row max of the raw scores (the scale is positive, so scaling after the
      // max gives the max of the scaled scores), over 8 interleaved partials:
      // short dependency chains instead of one chain through all 64 columns.
      float m8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) m8[e] = -1e30f;
#pragma unroll
      for (int c = 0; c < C::BN; ++c) m8[c & 7] = fmaxf(m8[c & 7], s[c]);
      const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * p.scale_log2;
      float alpha = 1.0f;
      if (j == 0) {
        m_used = mx;
      } else if (mx > m_used + kLazyRescaleLog2) {
        alpha = fast_exp2(m_used - mx);
        m_used = mx;
        l *= alpha;
      }
      float l8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) l8[e] = 0.f;
#pragma unroll
      for (int c = 0; c < C::BN; ++c) {
        const float e = fast_exp2(fmaf(s[c], p.scale_log2, -m_used));   // masked: 2^-inf = 0
        s[c] = e;
        l8[c & 7] += e;
      }
      l += ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
      if (j > 0) {
        // The previous P V of this tile has completed: P's columns are free and O may be rescaled.
        if (!__all_sync(0xffffffffu, wait_bar(&pv_done[tile], (j - 1) & 1, ctl, ERR_ATTN_FWD_WAIT))) { ok = false; break; }
        tc_fence_after();
        if (!__all_sync(0xffffffffu, alpha == 1.0f)) {
#pragma unroll 1
          for (int c = 0; c < DH / 32; ++c) {
            uint32_t rr[32];
            tmem_ld32(t_o + c * 32, rr);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
            tmem_st32(t_o + c * 32, rr);
          }
          tc_wait_st();
        }
      }
      {
        uint32_t pk[C::BN / 2];
#pragma unroll
        for (int g = 0; g < C::BN / 2; ++g) pk[g] = pack_f16x2(s[2 * g], s[2 * g + 1]);
        tmem_st32(t_p, pk);
        tc_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&p_full[tile]);
    }
    if (ok && n > 0 &&
        __all_sync(0xffffffffu, wait_bar(&pv_done[tile], (n - 1) & 1, ctl, ERR_ATTN_FWD_WAIT))) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const bool valid = q < p.S;
      uint16_t* orow = p.out + (long long)shard * p.T * p.Dt + ((long long)b * p.S + q) * p.Dt + hl * DH;
#pragma unroll 1
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(t_o + c * 32, rr);
        tc_wait_ld();
        if (valid) {
          float v[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(rr[e]) * inv_l;
#pragma unroll
          for (int g = 0; g < 4; ++g)
            *reinterpret_cast<uint4*>(orow + c * 32 + g * 8) = pack8_bf16(&v[g * 8]);
        }
      }
      if (valid) p.lse[((long long)b * p.H + h) * p.S + q] = (m_used + __log2f(l)) * kLn2;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// =====================================================================================
// Backward
// =====================================================================================
// Dv = rowsum(dO * O) and lse2 = lse * log2(e) for every (batch, head, query),
// written with rows padded to S_pad: padded queries get lse2 = +inf, Dv = 0.
// Block (x, y) covers queries [x * 16 * PREP_ROWS, ...) of batch-head y (b =
// y / H, h = y % H), so the head's shard and column offset are computed once
// per block.  dh/8 consecutive threads share one row (8 elements each, one
// 16-byte load of O and of dO) and reduce with shuffles, so a warp reads whole
// rows; a thread group's PREP_ROWS rows are loaded before any is reduced.
constexpr int PREP_ROWS = 4;

__global__ void __launch_bounds__(256)
attn_bwd_prep_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                     const float* __restrict__ lse, float* __restrict__ dvec,
                     float* __restrict__ lse2, int B, int S, int S_pad, int H, int Ht, int dh,
                     int Dt, long long T) {
  grid_dep_wait();
  grid_dep_launch();
  const int tpr = dh >> 3;                    // threads per row: 8 or 16
  const int rpb = blockDim.x / tpr;           // rows per group
  const int sub = threadIdx.x & (tpr - 1);
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh - b * H;
  const int shard = h / Ht, hl = h - shard * Ht;
  const long long head_base = (long long)shard * T * Dt + (long long)b * S * Dt + hl * dh + sub * 8;
  const long long vrow = (long long)bh * S_pad;
  const int s0 = blockIdx.x * rpb * PREP_ROWS + threadIdx.x / tpr;
  uint4 av[PREP_ROWS], gv[PREP_ROWS];
#pragma unroll
  for (int u = 0; u < PREP_ROWS; ++u) {
    const int s = s0 + u * rpb;
    if (s < S) {
      const long long off = head_base + (long long)s * Dt;
      av[u] = *reinterpret_cast<const uint4*>(o + off);
      gv[u] = *reinterpret_cast<const uint4*>(dout + off);
    }
  }
#pragma unroll
  for (int u = 0; u < PREP_ROWS; ++u) {
    const int s = s0 + u * rpb;
    float acc = 0.f;
    if (s < S) {
      const uint32_t wa[4] = {av[u].x, av[u].y, av[u].z, av[u].w};
      const uint32_t wg[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
        acc += bf16_lo(wa[k]) * f16_lo(wg[k]) + bf16_hi(wa[k]) * f16_hi(wg[k]);
    }
    for (int m = tpr >> 1; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (s < S_pad && sub == 0) {
      dvec[vrow + s] = s < S ? acc : 0.f;
      lse2[vrow + s] = s < S ? lse[(long long)bh * S + s] * kLog2e : INFINITY;
    }
  }
}

// ---------------------------------------------------------------- dK / dV
// Per 128-key block, walk 64-query blocks.  Two S^T/dP^T buffers in TMEM,
// one per compute warpgroup (block k uses buffer k % 2): the score MMAs of
// block k+1 and the dV/dK MMAs of block k-1 run while the compute warps work
// on block k.  P^T and dS^T (fp16) replace, in place, the halves of S^T and
// dP^T that have been copied out, and are the A operands of dV += P^T dO and
// dK += dS^T q.
template <int DH>
struct DkdvCfg {
  static constexpr int BK = 128, BQ = 64, CH = DH / 64;
  static constexpr int K_BYTES = BK * DH * 2;              // K and V tiles, each
  static constexpr int Q_BYTES = BQ * DH * 2;              // q and dO tiles, each (per stage)
  static constexpr int VEC_BYTES = BQ * 4;                 // lse2 / dvec slice of one stage
  static constexpr int STAGES = 3;                         // q / dO / lse2 / dvec ring depth
  static constexpr int STAGE_BYTES = 2 * Q_BYTES;
  static constexpr int OFF_K = 0, OFF_V = K_BYTES;
  static constexpr int OFF_ST = 2 * K_BYTES;               // stage s: q | dO
  static constexpr int DS_BYTES = 32 * BQ * 2;             // one compute warp's dS^T block (32 keys)
  static constexpr int OFF_DS = OFF_ST + STAGES * STAGE_BYTES;   // compute warp w at +w*DS_BYTES
  static constexpr int OFF_VEC = OFF_DS + 8 * DS_BYTES;    // stage s: lse2 at +2s*VEC, dvec at +(2s+1)*VEC
  static constexpr int OFF_BAR = OFF_VEC + STAGES * 2 * VEC_BYTES;
  static constexpr int RAW = OFF_BAR + 256 + 1024;
  static constexpr int SMEM = RAW > 120 * 1024 ? RAW : 120 * 1024;
};
static_assert(DkdvCfg<128>::SMEM <= 227 * 1024, "dK/dV tile exceeds shared memory");

// Work item i of the dK/dV launch: (key block, head, batch), the key block
// varying slowest, so that in item order the longest causal items come first.
struct DkdvItem {
  int kb, h, b;
};
__device__ __forceinline__ DkdvItem dkdv_item(int i, int H, int B) {
  const int hb = H * B;
  DkdvItem it;
  it.kb = i / hb;
  const int r = i - it.kb * hb;
  it.h = r % H;
  it.b = r / H;
  return it;
}

constexpr int DKDV_THREADS = 480;

// Persistent: one CTA per SM walks its items in snake order (snake_item).
// Warp roles: 0 loads (K/V per item, q/dO/lse2/Dv per 64-query block), 1
// issues the score products S^T = K q^T and dP^T = V dO^T, 2-9 are two
// compute warpgroups (P^T, dS^T), 10 issues dV += P^T dO and dK += dS^T q,
// 11-14 are the epilogue (dV, dK out of tensor memory to global, and their
// column partials).  The block counter g runs over all items of the CTA, so
// the stage ring and the two score buffers carry on from one item to the
// next: the next item's K/V load and first score products overlap the
// current item's last products and its epilogue, and the epilogue overlaps
// the next item's first blocks.  Per item: kv_full / kv_empty guard K and V
// (reloaded once the item's last score products completed), acc_full /
// acc_empty guard the dV/dK accumulators (the next item's first products wait
// until the epilogue warps have read them out).
template <int DH>
__global__ void __launch_bounds__(DKDV_THREADS, 1)
attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_kv128,
                     const __grid_constant__ CUtensorMap tm_q64,
                     const __grid_constant__ CUtensorMap tm_do64, const AttnArgs p) {
  using C = DkdvCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* qd_full = bars + 1;    // [STAGES <= 4] per stage
  uint64_t* qd_empty = bars + 5;   // [STAGES]
  uint64_t* s_full = bars + 9;     // [2] per TMEM buffer
  uint64_t* p_full = bars + 11;    // [2]
  uint64_t* mm2_done = bars + 13;  // [2]
  uint64_t* kv_empty = bars + 15;  // the item's score products completed: K/V reusable
  uint64_t* acc_full = bars + 16;  // the item's dV/dK complete
  uint64_t* acc_empty = bars + 17; // the epilogue has read dV/dK out
  uint64_t* drain = bars + 18;     // [2] each issuer's products completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 20);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = (p.S + C::BK - 1) / C::BK;
  const int nitems = nkb * p.H * p.B;
  const int nqb = (p.S + C::BQ - 1) / C::BQ;
  const Ctl ctl{abort_flag, p.err};
  // Per-item geometry.
  struct Geo {
    int b, bh, shard, k0, i0, nsteps, colq, colk, colv, cold;
    long long hrow;
  };
  auto geo = [&](int i) {
    const DkdvItem it = dkdv_item(i, p.H, p.B);
    Geo g;
    g.b = it.b;
    g.bh = it.b * p.H + it.h;
    g.shard = it.h / p.Ht;
    const int hl = it.h - g.shard * p.Ht;
    g.k0 = it.kb * C::BK;
    g.i0 = p.causal ? g.k0 / C::BQ : 0;
    g.nsteps = nqb - g.i0;
    g.colq = hl * DH;
    g.colk = p.Dt + hl * DH;
    g.colv = 2 * p.Dt + hl * DH;
    g.cold = hl * DH;
    g.hrow = ((long long)it.b * p.H + it.h) * p.S_pad;
    return g;
  };

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&qd_full[i], 1);
      mbar_init(&qd_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);   // buffer i belongs to compute warpgroup i
      mbar_init(&mm2_done[i], 1);
      mbar_init(&drain[i], 1);
    }
    mbar_init(kv_empty, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);        // one arrival per epilogue warp
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();   // inputs and outputs: the previous kernels have completed
  grid_dep_launch();
  // buffer j: S^T at 128j, dP^T at 128j + 64; dV at 256, dK at 384 (DH <= 128)
  const uint32_t t_dv = tmem + 256, t_dk = tmem + 256 + DH;

  if (warp == 0) {
    if (lane == 0) {
      int g = 0, n = 0, nkv = 0;
      bool ok = true;
      for (int rnd = 0; ok && (int)gridDim.x * rnd < nitems; ++rnd, ++n) {
        const int it = snake_item(rnd);
        if (it >= nitems) continue;
        const Geo q = geo(it);
        // K and V of the previous item are free once its score products completed.
        if (!(ok = wait_bar(kv_empty, (n & 1) ^ 1, ctl, ERR_ATTN_DKDV_WAIT))) break;
        mbar_arrive_expect_tx(kv_full, 2 * C::K_BYTES);
        for (int c = 0; c < C::CH; ++c) {
          tma_load_4d(smem + C::OFF_K + c * C::BK * 128, &tm_kv128, kv_full, q.colk + 64 * c, q.k0,
                      q.b, q.shard);
          tma_load_4d(smem + C::OFF_V + c * C::BK * 128, &tm_kv128, kv_full, q.colv + 64 * c, q.k0,
                      q.b, q.shard);
        }
        ++nkv;
        for (int k = 0; k < q.nsteps; ++k, ++g) {
          const int st = g % C::STAGES;
          const uint32_t u = g / C::STAGES;
          if (!(ok = wait_bar(&qd_empty[st], (u & 1) ^ 1, ctl, ERR_ATTN_DKDV_WAIT))) break;
          uint8_t* sq = smem + C::OFF_ST + st * C::STAGE_BYTES;
          uint8_t* sd = sq + C::Q_BYTES;
          uint8_t* sv = smem + C::OFF_VEC + st * 2 * C::VEC_BYTES;
          const int qs = (q.i0 + k) * C::BQ;
          mbar_arrive_expect_tx(&qd_full[st], 2 * C::Q_BYTES + 2 * C::VEC_BYTES);
          for (int c = 0; c < C::CH; ++c) {
            tma_load_4d(sq + c * C::BQ * 128, &tm_q64, &qd_full[st], q.colq + 64 * c, qs, q.b,
                        q.shard);
            tma_load_4d(sd + c * C::BQ * 128, &tm_do64, &qd_full[st], q.cold + 64 * c, qs, q.b,
                        q.shard);
          }
          bulk_load(sv, p.lse2 + q.hrow + qs, C::VEC_BYTES, &qd_full[st]);
          bulk_load(sv + C::VEC_BYTES, p.dvec + q.hrow + qs, C::VEC_BYTES, &qd_full[st]);
        }
      }
      // Copies still in flight land in this CTA's shared memory: wait for them
      // (bounded) before the CTA may exit: nkv K/V loads and stages 0 .. g-1.
      if (nkv > 0) mbar_wait(kv_full, (uint32_t)((nkv - 1) & 1), 200000000ull);
      for (int i = g - 1; i >= 0 && i >= g - C::STAGES; --i)
        mbar_wait(&qd_full[i % C::STAGES], (i / C::STAGES) & 1, 200000000ull);
    }
  } else if (warp == 1 || warp == 10) {
    // Two issuers, each blocking only on its own barriers: warp 1 issues
    // S^T/dP^T of block g (once its q/dO stage has landed and the dV/dK MMAs
    // of block g-2 have read P^T/dS^T out of the same buffer), warp 10 issues
    // dV/dK of block g (once its P^T/dS^T are in tensor memory) and releases
    // the stage.  Neither stream waits behind the other.
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_f32acc(128, C::BQ, false, false, true);
      constexpr uint32_t id_acc = idesc_f32acc(128, DH, false, true, true);
      const uint32_t sk = smem_u32(smem + C::OFF_K), sv = smem_u32(smem + C::OFF_V);
      int g = 0, n = 0;
      bool ok = true;
      if (warp == 1) {
        for (int rnd = 0; ok && (int)gridDim.x * rnd < nitems; ++rnd, ++n) {
          const int it = snake_item(rnd);
          if (it >= nitems) continue;
          const int nsteps = geo(it).nsteps;
          if (!(ok = wait_bar(kv_full, n & 1, ctl, ERR_ATTN_DKDV_WAIT))) break;
          for (int k = 0; k < nsteps; ++k, ++g) {
            const int bf = g & 1, st = g % C::STAGES;
            if (!(ok = wait_bar(&qd_full[st], (g / C::STAGES) & 1, ctl, ERR_ATTN_DKDV_WAIT))) break;
            if (!(ok = wait_bar(&mm2_done[bf], ((g >> 1) & 1) ^ 1, ctl, ERR_ATTN_DKDV_WAIT))) break;
            tc_fence_after();
            const uint32_t sq = smem_u32(smem + C::OFF_ST + st * C::STAGE_BYTES);
            const uint32_t sd = sq + C::Q_BYTES;
#pragma unroll
            for (int kk = 0; kk < DH / 16; ++kk) {
              tc_mma_f16(tmem + bf * 128, kmajor_desc(sk, C::BK, kk), kmajor_desc(sq, C::BQ, kk),
                         id_s, kk > 0);
              tc_mma_f16(tmem + bf * 128 + 64, kmajor_desc(sv, C::BK, kk),
                         kmajor_desc(sd, C::BQ, kk), id_s, kk > 0);
            }
            tc_commit(&s_full[bf]);
          }
          if (!ok) break;
          tc_commit(kv_empty);   // K/V may be reloaded once this item's score products completed
        }
        tc_commit(&drain[0]);
        mbar_wait(&drain[0], 0, 200000000ull);
      } else {
        for (int rnd = 0; ok && (int)gridDim.x * rnd < nitems; ++rnd, ++n) {
          const int it = snake_item(rnd);
          if (it >= nitems) continue;
          const int nsteps = geo(it).nsteps;
          // The first products of an item overwrite dV/dK: the epilogue has read the last item's.
          if (!(ok = wait_bar(acc_empty, (n & 1) ^ 1, ctl, ERR_ATTN_DKDV_WAIT))) break;
          for (int k = 0; k < nsteps; ++k, ++g) {
            const int bj = g & 1, sj = g % C::STAGES;
            if (!(ok = wait_bar(&p_full[bj], (g >> 1) & 1, ctl, ERR_ATTN_DKDV_WAIT))) break;
            tc_fence_after();
            const uint32_t sq = smem_u32(smem + C::OFF_ST + sj * C::STAGE_BYTES);
            const uint32_t sd = sq + C::Q_BYTES;
#pragma unroll
            for (int kk = 0; kk < C::BQ / 16; ++kk) {   // 16 queries = 8 columns per step
              tc_mma_f16_ts(t_dv, tmem + bj * 128 + 8 * kk, mnmajor_desc(sd, C::BQ, kk), id_acc,
                            (k | kk) != 0);
              tc_mma_f16_ts(t_dk, tmem + bj * 128 + 64 + 8 * kk, mnmajor_desc(sq, C::BQ, kk),
                            id_acc, (k | kk) != 0);
            }
            tc_commit(&mm2_done[bj]);
            tc_commit(&qd_empty[sj]);   // the scores of block g completed before its P^T existed
          }
          if (!ok) break;
          tc_commit(acc_full);
        }
        tc_commit(&drain[1]);
        mbar_wait(&drain[1], 0, 200000000ull);
      }
    }
  } else if (warp < 10) {
    // Two compute warpgroups: warpgroup w takes the blocks g with g % 2 == w
    // (its own TMEM buffer), so two blocks are in flight at once.
    const int wg = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint8_t* ds_buf = smem + C::OFF_DS + (warp - 2) * C::DS_BYTES;
    uint8_t* ds_row = ds_buf + lane * 128;
    int g0 = 0;   // first block counter of the current item
    bool ok = true;
    for (int rnd = 0; ok && (int)gridDim.x * rnd < nitems; ++rnd) {
      const int it = snake_item(rnd);
      if (it >= nitems) continue;
      const Geo q = geo(it);
      const int kpos = q.k0 + r;
      const bool kvalid = kpos < p.S;
      for (int k = ((g0 & 1) == wg) ? 0 : 1; k < q.nsteps; k += 2) {
        const int g = g0 + k;
        const int bf = g & 1;
        const uint32_t u = g >> 1;
        const int qs = (q.i0 + k) * C::BQ;
        if (!__all_sync(0xffffffffu, wait_bar(&s_full[bf], u & 1, ctl, ERR_ATTN_DKDV_WAIT))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* vl =
            reinterpret_cast<const float*>(smem + C::OFF_VEC + (g % C::STAGES) * 2 * C::VEC_BYTES);
        const float* vd = vl + C::BQ;
        // S^T and dP^T leave tensor memory in two 32-column halves; P^T and dS^T
        // of each half (fp16 pairs, 16 columns) are written back over the half
        // of S^T / dP^T just copied out.  The buffer was free once the dV/dK
        // MMAs of block g-2 completed, which the score MMAs of this block
        // already waited for.
        const uint32_t t_st = tmem + bf * 128 + lane_off;
        // The warp's dS^T buffer: its previous block's store has read it out.
        if (p.dst != nullptr) {
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
        }
        // Queries qs + qi with qi < qmin precede key kpos and are masked (causal):
        // a select per element, taken only in blocks where some key row of the
        // warp has a masked query (the causal diagonal).
        const int qmin = p.causal ? kpos - qs : 0;
        const bool masked = !__all_sync(0xffffffffu, qmin <= 0);
        auto half = [&](int c, auto mask_tag) {
          constexpr bool MASK = decltype(mask_tag)::value;
          uint32_t rs[32], rd[32];
          tmem_ld32(t_st + c * 32, rs);
          tmem_ld32(t_st + 64 + c * 32, rd);
          tc_wait_ld();
          uint32_t pk[16], dk[16];   // fp16 pairs of P^T and dS^T
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            // lse2 and Dv of four queries in one shared-memory load each.
            const float4 l4 = *reinterpret_cast<const float4*>(vl + c * 32 + e);
            const float4 d4 = *reinterpret_cast<const float4*>(vd + c * 32 + e);
            const float la[4] = {l4.x, l4.y, l4.z, l4.w}, da[4] = {d4.x, d4.y, d4.z, d4.w};
            float pe[4], de[4];
#pragma unroll
            for (int h4 = 0; h4 < 4; ++h4) {
              // Padded queries carry lse2 = +inf and dvec = 0, so they give 0.
              float x = fast_exp2(fmaf(__uint_as_float(rs[e + h4]), p.scale_log2, -la[h4]));
              if (MASK) x = c * 32 + e + h4 < qmin ? 0.f : x;
              pe[h4] = x;
              de[h4] = x * (__uint_as_float(rd[e + h4]) - da[h4]);
            }
            pk[e / 2] = pack_f16x2(pe[0], pe[1]);
            pk[e / 2 + 1] = pack_f16x2(pe[2], pe[3]);
            dk[e / 2] = pack_f16x2(de[0], de[1]);
            dk[e / 2 + 1] = pack_f16x2(de[2], de[3]);
          }
          tmem_st16(t_st + c * 16, pk);
          tmem_st16(t_st + 64 + c * 16, dk);
          if (p.dst != nullptr) {
            // dS^T row kpos (lane), queries 32c .. 32c+31 of the block: 16-byte
            // chunks 4c .. 4c+3 of the lane's 128-byte row, swizzled (zeros
            // for padded keys).
#pragma unroll
            for (int g4 = 0; g4 < 4; ++g4)
              *reinterpret_cast<uint4*>(ds_row + (((4 * c + g4) ^ (lane & 7)) << 4)) =
                  kvalid ? make_uint4(dk[4 * g4], dk[4 * g4 + 1], dk[4 * g4 + 2], dk[4 * g4 + 3])
                         : make_uint4(0u, 0u, 0u, 0u);
          }
        };
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          if (masked) half(c, BoolTag<true>{});
          else half(c, BoolTag<false>{});
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[bf]);
        if (p.dst != nullptr) {
          // The block's dS^T piece (32 keys x 64 queries) to global by one bulk copy.
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            const long long piece =
                ((long long)q.bh * (p.S_pad / 64) + qs / 64) * (p.S_pad / 32) + q.k0 / 32 + quad;
            bulk_store(p.dst + piece * 2048, ds_buf, C::DS_BYTES);
            bulk_commit();
          }
        }
      }
      g0 += q.nsteps;
    }
    if (p.dst != nullptr && lane == 0) bulk_wait0();
  } else {
    // Epilogue warps 11-14 (TMEM lane quarter warp % 4): dV and dK of each
    // item, once its last products completed, to global memory (fp16, dK
    // scaled by 1/sqrt(dh)) with their column partials for dbqkv; then the
    // accumulators are released to the next item.
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const long long w3 = 3LL * p.Dt;
    int n = 0;
    for (int rnd = 0; (int)gridDim.x * rnd < nitems; ++rnd, ++n) {
      const int it = snake_item(rnd);
      if (it >= nitems) continue;
      const Geo q = geo(it);
      if (!__all_sync(0xffffffffu, wait_bar(acc_full, n & 1, ctl, ERR_ATTN_DKDV_WAIT))) break;
      tc_fence_after();
      const int kpos = q.k0 + r;
      const bool valid = kpos < p.S;
      uint16_t* row = p.out + (long long)q.shard * p.T * w3 + ((long long)q.b * p.S + kpos) * w3;
#pragma unroll 1
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t rv[32], rk[32];
        tmem_ld32(t_dv + lane_off + c * 32, rv);
        tmem_ld32(t_dk + lane_off + c * 32, rk);
        tc_wait_ld();
        float v[32], kx[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          v[e] = valid ? __uint_as_float(rv[e]) : 0.f;
          kx[e] = valid ? __uint_as_float(rk[e]) * p.inv_sqrt_dh : 0.f;
        }
        if (valid) {
          bool over = false;
#pragma unroll
          for (int e = 0; e < 32; ++e) over |= fabsf(v[e]) > 65504.0f || fabsf(kx[e]) > 65504.0f;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            *reinterpret_cast<uint4*>(row + q.colv + c * 32 + g * 8) = pack8_f16(&v[g * 8]);
            *reinterpret_cast<uint4*>(row + q.colk + c * 32 + g * 8) = pack8_f16(&kx[g * 8]);
          }
          if (over && p.err) atomicCAS(p.err, 0u, 0x301u);
        }
        if (p.colpart != nullptr) {
          const int s0 = q.k0 + quad * 32;
          colpart_store(p, v, q.b, s0, q.shard, q.colv + c * 32);
          colpart_store(p, kx, q.b, s0, q.shard, q.colk + c * 32);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dQ
// Per 128-query block, walk 64-key blocks through a 4-stage K/V ring.  Two
// S/dP buffers in TMEM, one per compute warpgroup; dS (fp16 pairs) goes to
// its own TMEM columns and is the A operand of dQ += dS k.
//
// Persistent like the dK/dV kernel: one CTA per SM walks the (query block,
// head, batch) items longest first, in snake order (snake_item).  The block
// counter g runs across the CTA's items, so the K/V ring, the two S/dP
// buffers and the two dS buffers carry on from item to item; q/dO of the next
// item load once the item's last score products completed (q_empty), and the
// next item's first dQ products wait until four epilogue warps have read the
// accumulator out (acc_full / acc_empty).
template <int DH>
struct DqCfg {
  static constexpr int BQ = 128, BK = 64, CH = DH / 64;
  static constexpr int Q_BYTES = BQ * DH * 2;                // q and dO tiles, each
  static constexpr int K_BYTES = BK * DH * 2;                // K and V tiles, each (per stage)
  static constexpr int OFF_Q = 0, OFF_DO = Q_BYTES;
  static constexpr int STAGES = 4;                           // K / V ring depth
  static constexpr int OFF_ST = 2 * Q_BYTES;                 // stage s: k at +s*2*K, v at +K
  static constexpr int OFF_BAR = OFF_ST + STAGES * 2 * K_BYTES;
  static constexpr int RAW = OFF_BAR + 256 + 1024;
  static constexpr int SMEM = RAW > 120 * 1024 ? RAW : 120 * 1024;
};
static_assert(DqCfg<128>::SMEM <= 227 * 1024, "dQ tile exceeds shared memory");

constexpr int DQ_THREADS = 480;

template <int DH>
__global__ void __launch_bounds__(DQ_THREADS, 1)
attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q128,
                   const __grid_constant__ CUtensorMap tm_do128,
                   const __grid_constant__ CUtensorMap tm_kv64, const AttnArgs p) {
  using C = DqCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;    // [STAGES <= 4] per stage
  uint64_t* kv_empty = bars + 5;   // [STAGES]
  uint64_t* s_full = bars + 9;     // [2] per TMEM buffer
  uint64_t* s_free = bars + 11;    // [2]
  uint64_t* p_full = bars + 13;    // [2] per dS buffer
  uint64_t* mm2_done = bars + 15;  // [2]
  uint64_t* q_empty = bars + 17;   // the item's score products completed: q/dO reusable
  uint64_t* acc_full = bars + 18;  // the item's dQ complete
  uint64_t* acc_empty = bars + 19; // the epilogue has read dQ out
  uint64_t* drain = bars + 20;     // [2] each issuer's products completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 22);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (p.S + C::BQ - 1) / C::BQ;
  const int nkb = (p.S + C::BK - 1) / C::BK;
  const int nitems = nqb * p.H * p.B;
  const Ctl ctl{abort_flag, p.err};
  // Per-item geometry; items in (query block, head, batch) order with the
  // length index slowest, longest causal item first.
  struct Geo {
    int b, h, shard, q0, nsteps, colq, colk, colv, cold;
  };
  auto geo = [&](int i) {
    const int hb = p.H * p.B;
    const int x = i / hb;
    const int r = i - x * hb;
    Geo g;
    g.h = r % p.H;
    g.b = r / p.H;
    g.shard = g.h / p.Ht;
    const int hl = g.h - g.shard * p.Ht;
    const int qb = p.causal ? nqb - 1 - x : x;
    g.q0 = qb * C::BQ;
    g.nsteps = p.causal ? min(nkb, (g.q0 + C::BQ) / C::BK) : nkb;
    g.colq = hl * DH;
    g.colk = p.Dt + hl * DH;
    g.colv = 2 * p.Dt + hl * DH;
    g.cold = hl * DH;
    return g;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);   // buffer i belongs to compute warpgroup i
      mbar_init(&p_full[i], 128);
      mbar_init(&mm2_done[i], 1);
      mbar_init(&drain[i], 1);
    }
    mbar_init(q_empty, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);        // one arrival per epilogue warp
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();   // inputs and outputs: the previous kernels have completed
  grid_dep_launch();
  // TMEM columns: buffer j holds S at 128j, dP at 128j + 64 and dS (fp16 pairs)
  // at 384 + 32j; dQ accumulates at 256.
  const uint32_t t_dq = tmem + 256;

  if (warp == 0) {
    if (lane == 0) {
      int g = 0, n = 0, nq = 0;
      bool ok = true;
      for (int rnd = 0; ok && (int)gridDim.x * rnd < nitems; ++rnd, ++n) {
        const int it = snake_item(rnd);
        if (it >= nitems) continue;
        const Geo q = geo(it);
        // q and dO of the previous item are free once its score products completed.
        if (!(ok = wait_bar(q_empty, (n & 1) ^ 1, ctl, ERR_ATTN_DQ_WAIT))) break;
        mbar_arrive_expect_tx(q_full, 2 * C::Q_BYTES);
        for (int c = 0; c < C::CH; ++c) {
          tma_load_4d(smem + C::OFF_Q + c * C::BQ * 128, &tm_q128, q_full, q.colq + 64 * c, q.q0,
                      q.b, q.shard);
          tma_load_4d(smem + C::OFF_DO + c * C::BQ * 128, &tm_do128, q_full, q.cold + 64 * c, q.q0,
                      q.b, q.shard);
        }
        ++nq;
        for (int k = 0; k < q.nsteps; ++k, ++g) {
          const int st = g % C::STAGES;
          const uint32_t u = g / C::STAGES;
          if (!(ok = wait_bar(&kv_empty[st], (u & 1) ^ 1, ctl, ERR_ATTN_DQ_WAIT))) break;
          uint8_t* sk = smem + C::OFF_ST + st * 2 * C::K_BYTES;
          uint8_t* sv = sk + C::K_BYTES;
          mbar_arrive_expect_tx(&kv_full[st], 2 * C::K_BYTES);
          for (int c = 0; c < C::CH; ++c) {
            tma_load_4d(sk + c * C::BK * 128, &tm_kv64, &kv_full[st], q.colk + 64 * c, k * C::BK,
                        q.b, q.shard);
            tma_load_4d(sv + c * C::BK * 128, &tm_kv64, &kv_full[st], q.colv + 64 * c, k * C::BK,
                        q.b, q.shard);
          }
        }
      }
      // Copies still in flight land in this CTA's shared memory: wait for them
      // (bounded) before the CTA may exit: nq q/dO loads and stages 0 .. g-1.
      if (nq > 0) mbar_wait(q_full, (uint32_t)((nq - 1) & 1), 200000000ull);
      for (int i = g - 1; i >= 0 && i >= g - C::STAGES; --i)
        mbar_wait(&kv_full[i % C::STAGES], (i / C::STAGES) & 1, 200000000ull);
    }
  } else if (warp == 1 || warp == 10) {
    // Two issuers as in the dK/dV kernel: warp 1 issues S/dP of block g,
    // warp 10 dQ += dS K of block g and releases the K/V stage.
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_f32acc(128, C::BK, false, false, true);
      constexpr uint32_t id_acc = idesc_f32acc(128, DH, false, true, true);
      const uint32_t sq = smem_u32(smem + C::OFF_Q), sd = smem_u32(smem + C::OFF_DO);
      int g = 0, n = 0;
      bool ok = true;
      if (warp == 1) {
        for (int rnd = 0; ok && (int)gridDim.x * rnd < nitems; ++rnd, ++n) {
          const int it = snake_item(rnd);
          if (it >= nitems) continue;
          const int nsteps = geo(it).nsteps;
          if (!(ok = wait_bar(q_full, n & 1, ctl, ERR_ATTN_DQ_WAIT))) break;
          for (int k = 0; k < nsteps; ++k, ++g) {
            const int bf = g & 1, st = g % C::STAGES;
            if (!(ok = wait_bar(&kv_full[st], (g / C::STAGES) & 1, ctl, ERR_ATTN_DQ_WAIT))) break;
            if (!(ok = wait_bar(&s_free[bf], ((g >> 1) & 1) ^ 1, ctl, ERR_ATTN_DQ_WAIT))) break;
            tc_fence_after();
            const uint32_t sk = smem_u32(smem + C::OFF_ST + st * 2 * C::K_BYTES);
            const uint32_t sv = sk + C::K_BYTES;
#pragma unroll
            for (int kk = 0; kk < DH / 16; ++kk) {
              tc_mma_f16(tmem + bf * 128, kmajor_desc(sq, C::BQ, kk), kmajor_desc(sk, C::BK, kk),
                         id_s, kk > 0);
              tc_mma_f16(tmem + bf * 128 + 64, kmajor_desc(sd, C::BQ, kk),
                         kmajor_desc(sv, C::BK, kk), id_s, kk > 0);
            }
            tc_commit(&s_full[bf]);
          }
          if (!ok) break;
          tc_commit(q_empty);   // q/dO may be reloaded once this item's score products completed
        }
        tc_commit(&drain[0]);
        mbar_wait(&drain[0], 0, 200000000ull);
      } else {
        for (int rnd = 0; ok && (int)gridDim.x * rnd < nitems; ++rnd, ++n) {
          const int it = snake_item(rnd);
          if (it >= nitems) continue;
          const int nsteps = geo(it).nsteps;
          // The first products of an item overwrite dQ: the epilogue has read the last item's.
          if (!(ok = wait_bar(acc_empty, (n & 1) ^ 1, ctl, ERR_ATTN_DQ_WAIT))) break;
          for (int k = 0; k < nsteps; ++k, ++g) {
            const int bj = g & 1, sj = g % C::STAGES;
            if (!(ok = wait_bar(&p_full[bj], (g >> 1) & 1, ctl, ERR_ATTN_DQ_WAIT))) break;
            tc_fence_after();
            const uint32_t sk = smem_u32(smem + C::OFF_ST + sj * 2 * C::K_BYTES);
#pragma unroll
            for (int kk = 0; kk < C::BK / 16; ++kk)   // 16 keys = 8 columns of dS per step
              tc_mma_f16_ts(t_dq, tmem + 384 + 32 * bj + 8 * kk, mnmajor_desc(sk, C::BK, kk),
                            id_acc, (k | kk) != 0);
            tc_commit(&mm2_done[bj]);
            tc_commit(&kv_empty[sj]);   // the scores of block g completed before its dS existed
          }
          if (!ok) break;
          tc_commit(acc_full);
        }
        tc_commit(&drain[1]);
        mbar_wait(&drain[1], 0, 200000000ull);
      }
    }
  } else if (warp < 10) {
    // Two compute warpgroups: warpgroup w takes the blocks g with g % 2 == w
    // (its own S/dP and dS buffers), so two blocks are in flight at once.
    const int wg = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    int g0 = 0;   // first block counter of the current item
    bool ok = true;
    for (int rnd = 0; ok && (int)gridDim.x * rnd < nitems; ++rnd) {
      const int it = snake_item(rnd);
      if (it >= nitems) continue;
      const Geo q = geo(it);
      const int qr = q.q0 + r;
      const long long hrow = ((long long)q.b * p.H + q.h) * p.S_pad;
      const float l2 = p.lse2[hrow + qr];     // padded rows: +inf, so P = 0
      const float dv = p.dvec[hrow + qr];
      // Keys past the last visible one (after the query, or past S) are masked.
      const int klast = p.causal ? min(qr, p.S - 1) : p.S - 1;
      for (int k = ((g0 & 1) == wg) ? 0 : 1; k < q.nsteps; k += 2) {
        const int g = g0 + k;
        const int bf = g & 1;
        const uint32_t u = g >> 1;
        const int kmax = klast - k * C::BK;
        if (!__all_sync(0xffffffffu, wait_bar(&s_full[bf], u & 1, ctl, ERR_ATTN_DQ_WAIT))) {
          ok = false;
          break;
        }
        // The dS columns of buffer bf were last read by the dQ MMAs of block g-2.
        if (g >= 2 && !__all_sync(0xffffffffu, wait_bar(&mm2_done[bf], (u - 1) & 1, ctl,
                                                        ERR_ATTN_DQ_WAIT))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tb = tmem + bf * 128 + lane_off;
        // The select only where some row of the warp has a masked key.
        const bool masked = !__all_sync(0xffffffffu, kmax >= C::BK - 1);
        // S and dP leave tensor memory in two 32-key halves; the buffer goes
        // back to the score issuer once both halves are in registers, and dS of
        // each half (fp16 pairs, 16 columns) goes to this block's dS buffer.
        auto half = [&](int c, auto mask_tag) {
          constexpr bool MASK = decltype(mask_tag)::value;
          uint32_t rs[32], rd[32];
          tmem_ld32(tb + 32 * c, rs);
          tmem_ld32(tb + 64 + 32 * c, rd);
          tc_wait_ld();
          if (c == 1) {
            tc_fence_before();
            mbar_arrive(&s_free[bf]);
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float pe0 = fast_exp2(fmaf(__uint_as_float(rs[e]), p.scale_log2, -l2));
            float pe1 = fast_exp2(fmaf(__uint_as_float(rs[e + 1]), p.scale_log2, -l2));
            if (MASK) {
              pe0 = c * 32 + e > kmax ? 0.f : pe0;
              pe1 = c * 32 + e + 1 > kmax ? 0.f : pe1;
            }
            pk[e / 2] = pack_f16x2(pe0 * (__uint_as_float(rd[e]) - dv),
                                   pe1 * (__uint_as_float(rd[e + 1]) - dv));
          }
          tmem_st16(tmem + 384 + 32 * bf + lane_off + 16 * c, pk);
        };
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          if (masked) half(c, BoolTag<true>{});
          else half(c, BoolTag<false>{});
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[bf]);
      }
      g0 += q.nsteps;
    }
  } else {
    // Epilogue warps 11-14 (TMEM lane quarter warp % 4): dQ of each item,
    // once its last products completed, to global memory (fp16, scaled by
    // 1/sqrt(dh)) with its column partials for dbqkv; then the accumulator is
    // released to the next item.
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const long long w3 = 3LL * p.Dt;
    int n = 0;
    for (int rnd = 0; (int)gridDim.x * rnd < nitems; ++rnd, ++n) {
      const int it = snake_item(rnd);
      if (it >= nitems) continue;
      const Geo q = geo(it);
      if (!__all_sync(0xffffffffu, wait_bar(acc_full, n & 1, ctl, ERR_ATTN_DQ_WAIT))) break;
      tc_fence_after();
      const int qr = q.q0 + r;
      const bool qvalid = qr < p.S;
      uint16_t* row = p.out + (long long)q.shard * p.T * w3 + ((long long)q.b * p.S + qr) * w3 + q.colq;
#pragma unroll 1
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t rq[32];
        tmem_ld32(t_dq + lane_off + c * 32, rq);
        tc_wait_ld();
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = qvalid ? __uint_as_float(rq[e]) * p.inv_sqrt_dh : 0.f;
        if (qvalid) {
          bool over = false;
#pragma unroll
          for (int e = 0; e < 32; ++e) over |= fabsf(v[e]) > 65504.0f;
#pragma unroll
          for (int gg = 0; gg < 4; ++gg)
            *reinterpret_cast<uint4*>(row + c * 32 + gg * 8) = pack8_f16(&v[gg * 8]);
          if (over && p.err) atomicCAS(p.err, 0u, 0x301u);
        }
        if (p.colpart != nullptr) colpart_store(p, v, q.b, q.q0 + quad * 32, q.shard, q.colq + c * 32);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dQ from stored dS
// When the dK/dV kernel also stores dS^T (fp16, the same values it feeds to
// dK += dS^T q; AttnArgs::dst gives the layout), dQ = dS k needs no
// recomputation of S and dP: per 256-query block (two 128-row halves, each
// with its own accumulator), walk 64-key blocks through a 2-stage ring of
// (dS^T tile, k tile) and accumulate dQ += dS k with dS as an MN-major A
// operand (queries contiguous in each key row; bulk copies of 8 KiB,
// contiguous in global memory) and k as an MN-major B operand (TMA), each k
// tile serving both halves.  Under the causal mask the first half stops two
// key blocks before the second (dS^T past its diagonal was never written).
// Warp 0 loads, warp 1 issues the products, warps 2-9 (two per TMEM lane
// quarter, one per half) write dQ.  256 TMEM columns and 96 KB of shared
// memory: two CTAs share an SM, so one's epilogue overlaps the other's
// products.
template <int DH>
struct DqdsCfg {
  static constexpr int BQ = 256, BK = 64, CH = DH / 64, STAGES = 2;
  static constexpr int HALF_BYTES = 128 * BK * 2;            // dS^T of one half: 64 key rows x 128 queries
  static constexpr int A_BYTES = 2 * HALF_BYTES;
  static constexpr int K_BYTES = BK * DH * 2;                // k tile
  static constexpr int STAGE_BYTES = A_BYTES + K_BYTES;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr int THREADS = 320;
};

template <int DH>
__global__ void __launch_bounds__(320, 2)
attn_bwd_dq_ds_kernel(const __grid_constant__ CUtensorMap tm_kv64, const AttnArgs p) {
  using C = DqdsCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars + 0;       // [STAGES <= 3]
  uint64_t* empty = bars + 3;      // [STAGES]
  uint64_t* acc_full = bars + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 7);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (p.S + C::BQ - 1) / C::BQ;
  const AttnItem item = attn_item();
  const int qb = p.causal ? nqb - 1 - item.x : item.x;
  const int h = item.h, b = item.b;
  const int shard = h / p.Ht, hl = h - shard * p.Ht;
  const int q0 = qb * C::BQ;
  const int nkb = (p.S + C::BK - 1) / C::BK;
  // Key blocks of each half (a half wholly past S has none); the second
  // half's count is the block's.
  auto half_blocks = [&](int qs) {
    return qs >= p.S ? 0 : (p.causal ? min(nkb, (qs + 128) / C::BK) : nkb);
  };
  const int nk0 = half_blocks(q0), nk1 = half_blocks(q0 + 128);
  const int nsteps = max(nk0, nk1);
  const int colq = hl * DH, colk = p.Dt + hl * DH;
  const int bh = b * p.H + h;
  // dS^T pieces of this query block (its first 64-query column, key piece 0).
  const uint16_t* ds_col = p.dst + ((long long)bh * (p.S_pad / 64) + 4 * qb) * (p.S_pad / 32) * 2048;
  const Ctl ctl{abort_flag, p.err};

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_kv64);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t t_dq = *tmem_slot;   // half j at column 128 j
  grid_dep_wait();   // inputs and outputs: the previous kernels have completed
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      int k = 0;
      for (; k < nsteps; ++k) {
        const int st = k % C::STAGES;
        const uint32_t u = k / C::STAGES;
        if (!wait_bar(&empty[st], (u & 1) ^ 1, ctl, ERR_ATTN_DQ_WAIT)) break;
        uint8_t* sa = smem + st * C::STAGE_BYTES;
        uint8_t* sk = sa + C::A_BYTES;
        const bool a0 = k < nk0, a1 = k < nk1;
        mbar_arrive_expect_tx(&full[st], ((int)a0 + (int)a1) * C::HALF_BYTES + C::K_BYTES);
        // Each active half: two 64-query chunks of 64 key rows, two
        // consecutive 32-key pieces each.
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (!(j == 0 ? a0 : a1)) continue;
          for (int c = 0; c < 2; ++c)
            bulk_load(sa + j * C::HALF_BYTES + c * C::BK * 128,
                      ds_col + (long long)(2 * j + c) * (p.S_pad / 32) * 2048 + k * 4096,
                      C::BK * 128, &full[st]);
        }
        for (int c = 0; c < C::CH; ++c)
          tma_load_4d(sk + c * C::BK * 128, &tm_kv64, &full[st], colk + 64 * c, k * C::BK, b, shard);
      }
      for (int i = k - 1; i >= 0 && i >= k - C::STAGES; --i)
        mbar_wait(&full[i % C::STAGES], (i / C::STAGES) & 1, 200000000ull);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_acc = idesc_f32acc(128, DH, true, true, true);
      bool ok = true;
      for (int k = 0; ok && k < nsteps; ++k) {
        const int st = k % C::STAGES;
        if (!(ok = wait_bar(&full[st], (k / C::STAGES) & 1, ctl, ERR_ATTN_DQ_WAIT))) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + st * C::STAGE_BYTES);
        const uint32_t sk = sa + C::A_BYTES;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (k >= (j == 0 ? nk0 : nk1)) continue;
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk)   // 16 keys per product
            tc_mma_f16(t_dq + 128 * j, mnmajor_desc(sa + j * C::HALF_BYTES, C::BK, kk),
                       mnmajor_desc(sk, C::BK, kk), id_acc, (k | kk) != 0);
        }
        tc_commit(&empty[st]);
      }
      tc_commit(acc_full);   // also after an early stop: every issued product completes
      mbar_wait(acc_full, 0, 200000000ull);
    }
  } else {
    // Epilogue warps 2-9: half j = (warp - 2) / 4, TMEM lane quarter warp % 4.
    const int j = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int q = q0 + 128 * j + r;
    const bool qvalid = q < p.S;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    if ((j == 0 ? nk0 : nk1) > 0 && __all_sync(0xffffffffu, wait_bar(acc_full, 0, ctl, ERR_ATTN_DQ_WAIT))) {
      tc_fence_after();
      const long long w3 = 3LL * p.Dt;
      uint16_t* row = p.out + (long long)shard * p.T * w3 + ((long long)b * p.S + q) * w3 + colq;
#pragma unroll 1
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t rq[32];
        tmem_ld32(t_dq + 128 * j + lane_off + c * 32, rq);
        tc_wait_ld();
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = qvalid ? __uint_as_float(rq[e]) * p.inv_sqrt_dh : 0.f;
        if (qvalid) {
          bool over = false;
#pragma unroll
          for (int e = 0; e < 32; ++e) over |= fabsf(v[e]) > 65504.0f;
#pragma unroll
          for (int g = 0; g < 4; ++g)
            *reinterpret_cast<uint4*>(row + c * 32 + g * 8) = pack8_f16(&v[g * 8]);
          if (over && p.err) atomicCAS(p.err, 0u, 0x301u);
        }
        if (p.colpart != nullptr)
          colpart_store(p, v, b, q0 + 128 * j + quad * 32, shard, colq + c * 32);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(t_dq, 256);
  }
}

// =====================================================================================
// Host side
// =====================================================================================
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 4-D map over a shard-packed fp16 activation [t][B*S][width]: dims (width, S, B, t),
// box (64, rows, 1, 1), 128-byte swizzle, zero fill past S.
bool encode_act(CUtensorMap* m, const void* base, long long width, int S, int B, int t,
                long long T, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)width, (cuuint64_t)S, (cuuint64_t)B, (cuuint64_t)t};
  const cuuint64_t strides[3] = {(cuuint64_t)width * 2, (cuuint64_t)S * width * 2,
                                 (cuuint64_t)T * width * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// dS^T is kept for the dQ kernel when it takes at most this many bytes
// (attn_set_dst_limit; 4 GiB by default); larger problems recompute S and dP
// in the dQ kernel instead.
std::atomic<size_t> g_dst_max{size_t(4) << 30};

size_t dst_bytes(int B, int S, int H) {
  const size_t s_pad = ((size_t)S + 127) / 128 * 128;
  return (size_t)B * H * s_pad * s_pad * 2;
}

// A library call pins the limit for its thread (DstLimitPin), so that its
// workspace check, its carving and its launches all see one value.
thread_local bool t_dst_pinned = false;
thread_local size_t t_dst_limit = 0;

size_t dst_limit_now() { return t_dst_pinned ? t_dst_limit : g_dst_max.load(); }

bool keep_dst(int B, int S, int H) { return dst_bytes(B, S, H) <= dst_limit_now(); }

// Opt the kernel into `bytes` of dynamic shared memory once per device.
bool set_smem(const void* kern, int bytes) {
  static std::mutex mu;
  static const void* done[64][8] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  if (dev >= 0 && dev < 64)
    for (int i = 0; i < 8; ++i)
      if (done[dev][i] == kern) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  if (dev >= 0 && dev < 64)
    for (int i = 0; i < 8; ++i)
      if (!done[dev][i]) { done[dev][i] = kern; break; }
  return true;
}

// Query-key pairs that take part in the softmax (masked pairs not counted), all heads.
double core_pairs(const AttnArgs& a) {
  const double s = a.S;
  return (double)a.B * a.H * (a.causal ? s * (s + 1) / 2 : s * s);
}

AttnArgs make_args(int B, int S, int H, int dh, int t, int causal) {
  AttnArgs a{};
  a.B = B; a.S = S; a.H = H; a.Ht = H / t; a.Dt = (H / t) * dh; a.t = t;
  a.causal = causal;
  a.S_pad = (S + 127) / 128 * 128;
  a.T = (long long)B * S;
  a.scale_log2 = kLog2e / sqrtf((float)dh);
  a.inv_sqrt_dh = 1.0f / sqrtf((float)dh);
  a.err = error_word();
  return a;
}

template <int DH>
tp_status fwd_launch(const uint16_t* qkv, uint16_t* o, float* lse, const AttnArgs& a,
                     cudaStream_t st) {
  CUtensorMap tq, tkv;
  if (!encode_act(&tq, qkv, 3LL * a.Dt, a.S, a.B, a.t, a.T, 128) ||
      !encode_act(&tkv, qkv, 3LL * a.Dt, a.S, a.B, a.t, a.T, 64))
    return TP_ERR_CUDA;
  AttnArgs p = a;
  p.out = o;
  p.lse = lse;
  auto kern = attn_fwd_kernel<DH>;
  if (!set_smem((const void*)kern, FwdCfg<DH>::SMEM)) return TP_ERR_CUDA;
  const dim3 grid((a.S + 255) / 256, a.H, a.B);
  {
    TraceScope ts(st, TK_ATTN_FWD, 4.0 * DH * core_pairs(a));
    if (launch_pdl(kern, grid, dim3(FwdCfg<DH>::THREADS), FwdCfg<DH>::SMEM, st, tq, tkv, p) !=
        cudaSuccess)
      return TP_ERR_CUDA;
  }
  return cuda_status(cudaGetLastError());
}

template <int DH>
tp_status bwd_launch(const uint16_t* qkv, const uint16_t* o, const float* lse, const uint16_t* dout,
                     uint16_t* dqkv, const AttnArgs& a, void* scratch, cudaStream_t st) {
  float* dvec = static_cast<float*>(scratch);
  float* lse2 = dvec + (size_t)a.B * a.H * a.S_pad;
  {
    TraceScope ts(st, TK_ATTN_BWD_PREP);
    const int rows_per_block = 256 / (DH / 8) * PREP_ROWS;
    const dim3 grid((unsigned)((a.S_pad + rows_per_block - 1) / rows_per_block), (unsigned)(a.B * a.H));
    if (launch_pdl(attn_bwd_prep_kernel, grid, dim3(256), 0, st, o, dout, lse, dvec, lse2, a.B, a.S,
                   a.S_pad, a.H, a.Ht, DH, a.Dt, a.T) != cudaSuccess)
      return TP_ERR_CUDA;
  }
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  AttnArgs p = a;
  p.out = dqkv;
  p.lse2 = lse2;
  p.dvec = dvec;
  CUtensorMap kv128, q64, do64, q128, do128, kv64;
  if (!encode_act(&kv128, qkv, 3LL * a.Dt, a.S, a.B, a.t, a.T, 128) ||
      !encode_act(&q64, qkv, 3LL * a.Dt, a.S, a.B, a.t, a.T, 64) ||
      !encode_act(&do64, dout, a.Dt, a.S, a.B, a.t, a.T, 64) ||
      !encode_act(&q128, qkv, 3LL * a.Dt, a.S, a.B, a.t, a.T, 128) ||
      !encode_act(&do128, dout, a.Dt, a.S, a.B, a.t, a.T, 128) ||
      !encode_act(&kv64, qkv, 3LL * a.Dt, a.S, a.B, a.t, a.T, 64))
    return TP_ERR_CUDA;
  const bool with_dst = keep_dst(a.B, a.S, a.H);
  if (with_dst) p.dst = reinterpret_cast<uint16_t*>(lse2 + (size_t)a.B * a.H * a.S_pad);
  auto k1 = attn_bwd_dkdv_kernel<DH>;
  auto k2 = attn_bwd_dq_kernel<DH>;
  auto k3 = attn_bwd_dq_ds_kernel<DH>;
  if (!set_smem((const void*)k1, DkdvCfg<DH>::SMEM) ||
      !set_smem((const void*)(with_dst ? (const void*)k3 : (const void*)k2),
                with_dst ? DqdsCfg<DH>::SMEM : DqCfg<DH>::SMEM))
    return TP_ERR_CUDA;
  {
    // dP, dV and dK: three of the backward's four algorithmic products.
    TraceScope ts(st, TK_ATTN_BWD_DKDV, 6.0 * DH * core_pairs(a));
    // Persistent: one CTA per SM (at most one per work item).
    const long long items = (long long)((a.S + DkdvCfg<DH>::BK - 1) / DkdvCfg<DH>::BK) * a.H * a.B;
    const unsigned grid = (unsigned)(items < sm_count() ? items : sm_count());
    if (launch_pdl(k1, dim3(grid), dim3(DKDV_THREADS), DkdvCfg<DH>::SMEM, st, kv128, q64, do64, p) !=
        cudaSuccess)
      return TP_ERR_CUDA;
  }
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  if (with_dst) {
    TraceScope ts(st, TK_ATTN_BWD_DQ, 2.0 * DH * core_pairs(a));
    const dim3 grid((unsigned)((a.S + DqdsCfg<DH>::BQ - 1) / DqdsCfg<DH>::BQ), a.H, a.B);
    if (launch_pdl(k3, grid, dim3(DqdsCfg<DH>::THREADS), DqdsCfg<DH>::SMEM, st, kv64, p) !=
        cudaSuccess)
      return TP_ERR_CUDA;
    return cuda_status(cudaGetLastError());
  }
  {
    TraceScope ts(st, TK_ATTN_BWD_DQ, 2.0 * DH * core_pairs(a));
    // Persistent: one CTA per SM (at most one per work item).
    const long long items = (long long)((a.S + DqCfg<DH>::BQ - 1) / DqCfg<DH>::BQ) * a.H * a.B;
    const unsigned grid = (unsigned)(items < sm_count() ? items : sm_count());
    if (launch_pdl(k2, dim3(grid), dim3(DQ_THREADS), DqCfg<DH>::SMEM, st, q128, do128, kv64, p) !=
        cudaSuccess)
      return TP_ERR_CUDA;
  }
  return cuda_status(cudaGetLastError());
}

}  // namespace

tp_status launch_attn_fwd(const uint16_t* qkv, uint16_t* o, float* lse, int B, int S, int H,
                          int dh, int t, int causal, cudaStream_t stream) {
  if ((long long)B * S == 0) return TP_OK;
  const AttnArgs a = make_args(B, S, H, dh, t, causal);
  if (dh == 64) return fwd_launch<64>(qkv, o, lse, a, stream);
  if (dh == 128) return fwd_launch<128>(qkv, o, lse, a, stream);
  return TP_ERR_UNSUPPORTED;
}

size_t attn_set_dst_limit(size_t max_bytes) { return g_dst_max.exchange(max_bytes); }

DstLimitPin::DstLimitPin() : outer_(!t_dst_pinned) {
  if (outer_) {
    t_dst_limit = g_dst_max.load();
    t_dst_pinned = true;
  }
}

DstLimitPin::~DstLimitPin() {
  if (outer_) t_dst_pinned = false;
}

size_t attn_bwd_scratch_bytes(int B, int S, int H, int dh) {
  (void)dh;
  const size_t s_pad = ((size_t)S + 127) / 128 * 128;
  return 2 * (size_t)B * H * s_pad * sizeof(float) + (keep_dst(B, S, H) ? dst_bytes(B, S, H) : 0);
}

tp_status launch_attn_bwd(const uint16_t* qkv, const uint16_t* o, const float* lse,
                          const uint16_t* dout, uint16_t* dqkv, int B, int S, int H, int dh, int t,
                          int causal, void* scratch, cudaStream_t stream, float* colpart) {
  if ((long long)B * S == 0) return TP_OK;
  AttnArgs a = make_args(B, S, H, dh, t, causal);
  a.colpart = colpart;
  if (dh == 64) return bwd_launch<64>(qkv, o, lse, dout, dqkv, a, scratch, stream);
  if (dh == 128) return bwd_launch<128>(qkv, o, lse, dout, dqkv, a, scratch, stream);
  return TP_ERR_UNSUPPORTED;
}

}  // namespace tp
