// Rank-local entry points: ONE shard of the tensor-parallel sublayer per GPU.
//
// The pages' deployment ("One Idea, Two Insertions"; "How transformer layers
// actually decompose"; "Why TP must stay within a node") runs shard i of every
// weight on GPU i and joins the shards with one all-reduce per sublayer per
// direction: after the row-parallel product in the forward pass (the sum of
// the partial outputs H_i W2_i, O_i Wout_i) and after the column-parallel
// input gradient in the backward pass (the sum of dA_i W1_i^T, dqkv_i Wqkv_i^T).
// Each call here runs everything of ONE shard between two of those exchange
// points and writes its partial of the exchanged tensor in fp32, with no bias:
//
//   tp_mlp_fwd_rank   A_i, H_i = GeLU(x W1_i + b1_i);  partial = H_i W2_i
//   tp_mlp_bwd_rank   dA_i, dW2_i, dW1_i, db1_i (db2);  partial = dA_i W1_i^T
//   tp_attn_fwd_rank  qkv_i, per-head attention of the shard's heads (O_i,
//                     lse_i);  partial = O_i Wout_i
//   tp_attn_bwd_rank  dWout_i, the attention backward, dWqkv_i, dbqkv_i (dbout);
//                     partial = dqkv_i Wqkv_i^T
//
// The exchange itself is the caller's (an all-reduce among the t ranks, or
// reads of the peers' partials); tp_rowpar_finish then rounds the sum once,
// adding the bias of the row-parallel product once and the residual:
//   out = bf16( sum_p parts[p] + bias + resid )
// Summing the t partials in rank order gives a deterministic result that
// differs from the one-GPU library's only by the grouping of fp32 additions
// (there the shard walk accumulates every shard into one accumulator).
#include <cuda_runtime.h>

#include "gemm_sm100.cuh"
#include "internal.h"

namespace tp {

namespace {

using bf16p = const uint16_t*;

OperandDesc opnd(const void* p, bool mn, long long inner, long long outer, bool f16 = false) {
  // One unsharded operand: the rank holds only its own shard.
  return OperandDesc{p, mn, f16, SHARD_NONE, inner, outer, 1, inner, 0};
}

GemmProblem problem(long long M, long long N, long long K) {
  GemmProblem g{};
  g.m_shards = 1; g.n_shards = 1; g.Mt = (int)M; g.Nt = (int)N;
  g.k_shards = 1; g.Kt = (int)K;
  g.epi = EPI_LINEAR;
  g.ldc = N;
  return g;
}

struct RankSizes {
  long long B, S, T, D, H, dh, t, Hl, Dt, Ft;
};

RankSizes rank_sizes(const tp_dims& d) {
  RankSizes z{};
  z.B = d.batch; z.S = d.seq; z.T = (long long)d.batch * d.seq;
  z.D = d.hidden; z.H = d.heads; z.dh = d.head_dim; z.t = d.t;
  z.Hl = d.t > 0 ? d.heads / d.t : 0;
  z.Dt = d.t > 0 ? d.hidden / d.t : 0;
  z.Ft = d.t > 0 ? d.ffn / d.t : 0;
  return z;
}

size_t mlp_bwd_rank_ws(const RankSizes& z) {
  Carver c(nullptr);
  c.take<uint16_t>((size_t)(z.T * z.Ft));                 // dA_i
  c.take<float>(colsum_partial_floats(1, z.T, z.D));      // db2
  c.take<float>((size_t)((z.T + 31) / 32 * z.Ft));        // db1_i: a partial row per 32 rows
  return align_up(c.off, 256);
}

// fp16 copies of x (unless given) and of Wqkv_i: the attention sublayer's
// products run on fp16 operands.
size_t attn_fwd_rank_ws(const RankSizes& z) {
  Carver c(nullptr);
  c.take<uint16_t>((size_t)(z.T * z.D));
  c.take<uint16_t>((size_t)(z.D * 3 * z.Dt));
  return align_up(c.off, 256);
}

size_t attn_bwd_rank_ws(const RankSizes& z) {
  Carver c(nullptr);
  c.take<uint8_t>(attn_fwd_rank_ws(z));
  c.take<uint16_t>((size_t)(z.T * z.Dt));                 // dO_i (fp16)
  c.take<uint16_t>((size_t)(z.T * 3 * z.Dt));             // dqkv_i (fp16)
  c.take<uint8_t>(attn_bwd_scratch_bytes((int)z.B, (int)z.S, (int)z.Hl, (int)z.dh));
  c.take<float>(colsum_partial_floats(1, z.T, z.D));                  // dbout
  c.take<float>((size_t)(attn_colpart_rows(z.B, z.S) * 3 * z.Dt));    // dbqkv_i
  return align_up(c.off, 256);
}

// ---------------------------------------------------------------- finish kernel
constexpr int kMaxParts = 8;

struct FinishArgs {
  const float* parts[kMaxParts];
  int nparts;
  const uint16_t* bias;    // [cols] bf16, or null
  const uint16_t* resid;   // [rows][cols] bf16, or null
  uint16_t* out;           // [rows][cols] bf16
  float* out32;            // [rows][cols] fp32 copy, or null
  long long n8;            // rows * cols / 8
  int cols8;               // cols / 8
};

__global__ void __launch_bounds__(256) rowpar_finish_kernel(const FinishArgs a) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < a.n8;
       i += (long long)gridDim.x * blockDim.x) {
    float v[8];
    {
      const float4* p = reinterpret_cast<const float4*>(a.parts[0]) + 2 * i;
      const float4 lo = p[0], hi = p[1];
      v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
      v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
    }
    for (int k = 1; k < a.nparts; ++k) {   // rank order: a fixed summation order
      const float4* p = reinterpret_cast<const float4*>(a.parts[k]) + 2 * i;
      const float4 lo = p[0], hi = p[1];
      v[0] += lo.x; v[1] += lo.y; v[2] += lo.z; v[3] += lo.w;
      v[4] += hi.x; v[5] += hi.y; v[6] += hi.z; v[7] += hi.w;
    }
    if (a.bias != nullptr) {
      const uint4 b = reinterpret_cast<const uint4*>(a.bias)[i % a.cols8];
      const uint32_t w[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[2 * q] += bf16_lo(w[q]);
        v[2 * q + 1] += bf16_hi(w[q]);
      }
    }
    if (a.resid != nullptr) {
      const uint4 r = reinterpret_cast<const uint4*>(a.resid)[i];
      const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[2 * q] += bf16_lo(w[q]);
        v[2 * q + 1] += bf16_hi(w[q]);
      }
    }
    uint4 o;
    o.x = pack_bf16x2(v[0], v[1]);
    o.y = pack_bf16x2(v[2], v[3]);
    o.z = pack_bf16x2(v[4], v[5]);
    o.w = pack_bf16x2(v[6], v[7]);
    reinterpret_cast<uint4*>(a.out)[i] = o;
    if (a.out32 != nullptr) {
      float4* q = reinterpret_cast<float4*>(a.out32) + 2 * i;
      q[0] = make_float4(v[0], v[1], v[2], v[3]);
      q[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
}

}  // namespace

}  // namespace tp

using namespace tp;

extern "C" {

size_t tp_rank_workspace_size(int op, const tp_dims* dims) {
  DstLimitPin pin;   // one dS^T limit for the whole call
  switch (op) {
    case TP_RANK_MLP_FWD: return 0;
    case TP_RANK_MLP_BWD: return check_mlp(dims) == TP_OK ? mlp_bwd_rank_ws(rank_sizes(*dims)) : 0;
    case TP_RANK_ATTN_FWD:
      return check_attn(dims) == TP_OK ? attn_fwd_rank_ws(rank_sizes(*dims)) : 0;
    case TP_RANK_ATTN_BWD:
      return check_attn(dims) == TP_OK ? attn_bwd_rank_ws(rank_sizes(*dims)) : 0;
  }
  return 0;
}

tp_status tp_rowpar_finish(const float* const* parts, int nparts, const tp_bf16* bias,
                           const tp_bf16* resid, int rows, int cols, tp_bf16* out, float* out32,
                           tp_stream stream) {
  if (parts == nullptr || out == nullptr || rows < 0 || cols <= 0) return TP_ERR_INVALID_ARG;
  if (nparts < 1 || nparts > kMaxParts) return TP_ERR_INVALID_ARG;
  if (cols % 8) return TP_ERR_MISALIGNED;
  FinishArgs a{};
  for (int k = 0; k < nparts; ++k) {
    if (parts[k] == nullptr) return TP_ERR_INVALID_ARG;
    if (!al16(parts[k])) return TP_ERR_MISALIGNED;
    a.parts[k] = parts[k];
  }
  if (!all_aligned(bias, resid, out, out32)) return TP_ERR_MISALIGNED;
  if (rows == 0) return TP_OK;
  a.nparts = nparts;
  a.bias = bias;
  a.resid = resid;
  a.out = out;
  a.out32 = out32;
  a.n8 = (long long)rows * cols / 8;
  a.cols8 = cols / 8;
  long long blocks = (a.n8 + 255) / 256;
  if (blocks > 8LL * sm_count()) blocks = 8LL * sm_count();
  cudaStream_t st = (cudaStream_t)stream;
  {
    TraceScope ts(st, TK_FINISH);
    rowpar_finish_kernel<<<(unsigned)blocks, 256, 0, st>>>(a);
  }
  return cuda_status(cudaGetLastError());
}

// ---------------------------------------------------------------- MLP
tp_status tp_mlp_fwd_rank(const tp_dims* dims, const tp_bf16* x, const tp_bf16* w1_i,
                          const tp_bf16* b1_i, const tp_bf16* w2_i, tp_bf16* a_i, tp_bf16* h_i,
                          float* partial, tp_stream stream) {
  tp_status st = check_mlp(dims);
  if (st != TP_OK) return st;
  const RankSizes z = rank_sizes(*dims);
  if (!all_set(w1_i, w2_i) || (z.T > 0 && !all_set(x, a_i, h_i, partial)))
    return TP_ERR_INVALID_ARG;
  if (!all_aligned(x, w1_i, b1_i, w2_i, a_i, h_i, partial)) return TP_ERR_MISALIGNED;
  if (z.T == 0) return TP_OK;
  cudaStream_t cs = (cudaStream_t)stream;
  // Column-parallel: A_i = x W1_i + b1_i, H_i = GeLU(A_i) (local to the shard).
  GemmProblem g1 = problem(z.T, z.Ft, z.D);
  g1.a = opnd(x, false, z.D, z.T);
  g1.b = opnd(w1_i, true, z.Ft, z.D);
  g1.epi = EPI_BIAS_GELU; g1.c = a_i; g1.c2 = h_i; g1.bias = b1_i;
  if ((st = launch_gemm(g1, cs)) != TP_OK) return st;
  // Row-parallel partial: H_i W2_i in fp32, no bias (added once after the sum).
  GemmProblem g2 = problem(z.T, z.D, z.Ft);
  g2.a = opnd(h_i, false, z.Ft, z.T);
  g2.b = opnd(w2_i, true, z.D, z.Ft);
  g2.c = partial; g2.out_f32 = true;
  return launch_gemm(g2, cs);
}

tp_status tp_mlp_bwd_rank(const tp_dims* dims, const tp_bf16* x, const tp_bf16* w1_i,
                          const tp_bf16* w2_i, const tp_bf16* a_i, const tp_bf16* h_i,
                          const tp_bf16* dy, tp_bf16* dw1_i, tp_bf16* dw2_i, tp_bf16* db1_i,
                          tp_bf16* db2, float* partial, void* ws, size_t ws_bytes,
                          tp_stream stream) {
  tp_status st = check_mlp(dims);
  if (st != TP_OK) return st;
  const RankSizes z = rank_sizes(*dims);
  if (!all_set(w1_i, w2_i, dw1_i, dw2_i) || (z.T > 0 && !all_set(x, a_i, h_i, dy, partial)))
    return TP_ERR_INVALID_ARG;
  if (!all_aligned(x, w1_i, w2_i, a_i, h_i, dy, dw1_i, dw2_i, db1_i, db2, partial))
    return TP_ERR_MISALIGNED;
  cudaStream_t cs = (cudaStream_t)stream;
  if (z.T == 0) {
    cudaMemsetAsync(dw1_i, 0, (size_t)(z.D * z.Ft) * 2, cs);
    cudaMemsetAsync(dw2_i, 0, (size_t)(z.D * z.Ft) * 2, cs);
    if (db1_i) cudaMemsetAsync(db1_i, 0, (size_t)z.Ft * 2, cs);
    if (db2) cudaMemsetAsync(db2, 0, (size_t)z.D * 2, cs);
    return cuda_status(cudaGetLastError());
  }
  if ((st = check_ws(ws, ws_bytes, mlp_bwd_rank_ws(z))) != TP_OK) return st;
  Carver c(ws);
  uint16_t* da = c.take<uint16_t>((size_t)(z.T * z.Ft));
  float* part = c.take<float>(colsum_partial_floats(1, z.T, z.D));
  float* dapart = c.take<float>((size_t)((z.T + 31) / 32 * z.Ft));
  // dA_i = (dy W2_i^T) * GeLU'(A_i): W2_i [Ft][D] read as [n = Ft][k = D], K-major;
  // its epilogue also writes the column-sum partials of dA_i for db1_i.
  GemmProblem g4 = problem(z.T, z.Ft, z.D);
  g4.a = opnd(dy, false, z.D, z.T);
  g4.b = opnd(w2_i, false, z.D, z.Ft);
  g4.epi = EPI_DGELU; g4.c = da; g4.aux = a_i;
  if (db1_i) g4.colpart = dapart;
  if ((st = launch_gemm(g4, cs)) != TP_OK) return st;
  if (db1_i && (st = launch_colsum_reduce(dapart, (z.T + 31) / 32, z.Ft, db1_i, cs)) != TP_OK)
    return st;
  // dW2_i = H_i^T dy.
  GemmProblem g5 = problem(z.Ft, z.D, z.T);
  g5.a = opnd(h_i, true, z.Ft, z.T);
  g5.b = opnd(dy, true, z.D, z.T);
  g5.c = dw2_i;
  if ((st = launch_gemm(g5, cs)) != TP_OK) return st;
  // dW1_i = x^T dA_i.
  GemmProblem g6 = problem(z.D, z.Ft, z.T);
  g6.a = opnd(x, true, z.D, z.T);
  g6.b = opnd(da, true, z.Ft, z.T);
  g6.c = dw1_i;
  if ((st = launch_gemm(g6, cs)) != TP_OK) return st;
  // Partial of dx: dA_i W1_i^T in fp32 (W1_i [D][Ft] read as [n = D][k = Ft]).
  GemmProblem g7 = problem(z.T, z.D, z.Ft);
  g7.a = opnd(da, false, z.Ft, z.T);
  g7.b = opnd(w1_i, false, z.Ft, z.D);
  g7.c = partial; g7.out_f32 = true;
  if ((st = launch_gemm(g7, cs)) != TP_OK) return st;
  if (db2 && (st = launch_colsum_stacked(dy, 1, z.T, z.D, db2, part, cs)) != TP_OK) return st;
  return TP_OK;
}

// ---------------------------------------------------------------- attention
// The shard's heads are attended as a problem of H/t heads with t = 1: the
// shard's qkv_i [T][3Dt] is [q_i | k_i | v_i], local head j at j*dh of each.
static tp_status attn_inputs16(const RankSizes& z, const tp_bf16* x, const tp_f16* x16,
                               const tp_bf16* wqkv_i, Carver& c, const uint16_t** xo,
                               uint16_t** wo, cudaStream_t cs) {
  uint16_t* xc = c.take<uint16_t>((size_t)(z.T * z.D));
  uint16_t* w16 = c.take<uint16_t>((size_t)(z.D * 3 * z.Dt));
  tp_status st;
  if (x16 == nullptr) {
    if ((st = launch_cast_f16(x, (size_t)(z.T * z.D), xc, cs)) != TP_OK) return st;
    *xo = xc;
  } else {
    *xo = x16;
  }
  if ((st = launch_cast_f16(wqkv_i, (size_t)(z.D * 3 * z.Dt), w16, cs)) != TP_OK) return st;
  *wo = w16;
  return TP_OK;
}

tp_status tp_attn_fwd_rank(const tp_dims* dims, const tp_bf16* x, const tp_f16* x16,
                           const tp_bf16* wqkv_i, const tp_bf16* bqkv_i, const tp_bf16* wout_i,
                           tp_f16* qkv_i, tp_bf16* o_i, float* lse_i, float* partial, void* ws,
                           size_t ws_bytes, tp_stream stream) {
  tp_status st = check_attn(dims);
  if (st != TP_OK) return st;
  const RankSizes z = rank_sizes(*dims);
  if (!all_set(wqkv_i, wout_i) ||
      (z.T > 0 && (!all_set(qkv_i, o_i, lse_i, partial) || (x == nullptr) == (x16 == nullptr))))
    return TP_ERR_INVALID_ARG;
  if (!all_aligned(x, x16, wqkv_i, bqkv_i, wout_i, qkv_i, o_i, lse_i, partial))
    return TP_ERR_MISALIGNED;
  if (z.T == 0) return TP_OK;
  if ((st = check_ws(ws, ws_bytes, attn_fwd_rank_ws(z))) != TP_OK) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  Carver c(ws);
  const uint16_t* xin = nullptr;
  uint16_t* w16 = nullptr;
  if ((st = attn_inputs16(z, x, x16, wqkv_i, c, &xin, &w16, cs)) != TP_OK) return st;
  // Column-parallel by head: qkv_i = x Wqkv_i + bqkv_i (fp16).
  const long long w3 = 3 * z.Dt;
  GemmProblem g1 = problem(z.T, w3, z.D);
  g1.a = opnd(xin, false, z.D, z.T, true);
  g1.b = opnd(w16, true, w3, z.D, true);
  g1.c = qkv_i; g1.bias = bqkv_i; g1.out_f16 = true;
  if ((st = launch_gemm(g1, cs)) != TP_OK) return st;
  // Attention of the shard's H/t heads, local to the rank.
  if ((st = launch_attn_fwd(qkv_i, o_i, lse_i, (int)z.B, (int)z.S, (int)z.Hl, (int)z.dh, 1,
                            dims->causal, cs)) != TP_OK)
    return st;
  // Row-parallel partial: O_i Wout_i in fp32, no bias.
  GemmProblem g2 = problem(z.T, z.D, z.Dt);
  g2.a = opnd(o_i, false, z.Dt, z.T);
  g2.b = opnd(wout_i, true, z.D, z.Dt);
  g2.c = partial; g2.out_f32 = true;
  return launch_gemm(g2, cs);
}

tp_status tp_attn_bwd_rank(const tp_dims* dims, const tp_bf16* x, const tp_f16* x16,
                           const tp_bf16* wqkv_i, const tp_bf16* wout_i, const tp_f16* qkv_i,
                           const tp_bf16* o_i, const float* lse_i, const tp_bf16* dy,
                           tp_bf16* dwqkv_i, tp_bf16* dbqkv_i, tp_bf16* dwout_i, tp_bf16* dbout,
                           float* partial, void* ws, size_t ws_bytes, tp_stream stream) {
  DstLimitPin pin;   // one dS^T limit for the whole call
  tp_status st = check_attn(dims);
  if (st != TP_OK) return st;
  const RankSizes z = rank_sizes(*dims);
  const long long w3 = 3 * z.Dt;
  if (!all_set(wqkv_i, wout_i, dwqkv_i, dwout_i) ||
      (z.T > 0 && (!all_set(qkv_i, o_i, lse_i, dy, partial) || (x == nullptr) == (x16 == nullptr))))
    return TP_ERR_INVALID_ARG;
  if (!all_aligned(x, x16, wqkv_i, wout_i, qkv_i, o_i, lse_i, dy, dwqkv_i, dbqkv_i, dwout_i,
                   dbout, partial))
    return TP_ERR_MISALIGNED;
  cudaStream_t cs = (cudaStream_t)stream;
  if (z.T == 0) {
    cudaMemsetAsync(dwqkv_i, 0, (size_t)(z.D * w3) * 2, cs);
    cudaMemsetAsync(dwout_i, 0, (size_t)(z.Dt * z.D) * 2, cs);
    if (dbqkv_i) cudaMemsetAsync(dbqkv_i, 0, (size_t)w3 * 2, cs);
    if (dbout) cudaMemsetAsync(dbout, 0, (size_t)z.D * 2, cs);
    return cuda_status(cudaGetLastError());
  }
  if ((st = check_ws(ws, ws_bytes, attn_bwd_rank_ws(z))) != TP_OK) return st;
  Carver c(ws);
  const uint16_t* xin = nullptr;
  uint16_t* w16 = nullptr;
  if ((st = attn_inputs16(z, x, x16, wqkv_i, c, &xin, &w16, cs)) != TP_OK) return st;
  c.off = align_up(attn_fwd_rank_ws(z), 256);
  uint16_t* dout = c.take<uint16_t>((size_t)(z.T * z.Dt));
  uint16_t* dqkv = c.take<uint16_t>((size_t)(z.T * w3));
  void* scratch = c.take<uint8_t>(attn_bwd_scratch_bytes((int)z.B, (int)z.S, (int)z.Hl, (int)z.dh));
  float* part = c.take<float>(colsum_partial_floats(1, z.T, z.D));
  float* qkvpart = c.take<float>((size_t)(attn_colpart_rows(z.B, z.S) * w3));
  // dO_i = dy Wout_i^T (fp16): Wout_i [Dt][D] read as [n = Dt][k = D].
  GemmProblem g1 = problem(z.T, z.Dt, z.D);
  g1.a = opnd(dy, false, z.D, z.T);
  g1.b = opnd(wout_i, false, z.D, z.Dt);
  g1.c = dout; g1.out_f16 = true;
  if ((st = launch_gemm(g1, cs)) != TP_OK) return st;
  // dWout_i = O_i^T dy.
  GemmProblem g2 = problem(z.Dt, z.D, z.T);
  g2.a = opnd(o_i, true, z.Dt, z.T);
  g2.b = opnd(dy, true, z.D, z.T);
  g2.c = dwout_i;
  if ((st = launch_gemm(g2, cs)) != TP_OK) return st;
  if ((st = launch_attn_bwd(qkv_i, o_i, lse_i, dout, dqkv, (int)z.B, (int)z.S, (int)z.Hl,
                            (int)z.dh, 1, dims->causal, scratch, cs,
                            dbqkv_i ? qkvpart : nullptr)) != TP_OK)
    return st;
  if (dbqkv_i && (st = launch_colsum_reduce(qkvpart, attn_colpart_rows(z.B, z.S), w3, dbqkv_i,
                                            cs)) != TP_OK)
    return st;
  // dWqkv_i = x^T dqkv_i (fp16 operands).
  GemmProblem g3 = problem(z.D, w3, z.T);
  g3.a = opnd(xin, true, z.D, z.T, true);
  g3.b = opnd(dqkv, true, w3, z.T, true);
  g3.c = dwqkv_i;
  if ((st = launch_gemm(g3, cs)) != TP_OK) return st;
  // Partial of dx: dqkv_i Wqkv_i^T in fp32 (fp16 operands).
  GemmProblem g4 = problem(z.T, z.D, w3);
  g4.a = opnd(dqkv, false, w3, z.T, true);
  g4.b = opnd(w16, false, w3, z.D, true);
  g4.c = partial; g4.out_f32 = true;
  if ((st = launch_gemm(g4, cs)) != TP_OK) return st;
  if (dbout && (st = launch_colsum_stacked(dy, 1, z.T, z.D, dbout, part, cs)) != TP_OK) return st;
  return TP_OK;
}

}  // extern "C"
