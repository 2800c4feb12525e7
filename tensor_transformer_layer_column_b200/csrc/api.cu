// C ABI of libtplayer.so: argument validation, workspace carving and the
// sequencing of kernels for each sublayer (see include/tp_layer.h).
//
// The tensor-parallel structure (Megatron-LM pages, "How transformer layers
// actually decompose" and "The attention heads split") maps onto the GEMM's
// shard descriptors:
//   column-parallel product  (x W1_i, x Wqkv_i)      -> N shards, one launch for all t
//   row-parallel product + all-reduce (sum_i H_i W2_i) -> K shards into one accumulator
//   input-gradient reduction (sum_i dA_i W1_i^T)      -> K shards into one accumulator
//   weight gradients (H_i^T dY, x^T dA_i)             -> M or N shards
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "gemm_sm100.cuh"
#include "internal.h"

namespace tp {

__device__ unsigned int g_error_word;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned int* g_err_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

}  // namespace

unsigned int* error_word() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) == cudaSuccess)
      g_err_ptr[d] = static_cast<unsigned int*>(p);
  }
  return g_err_ptr[d];
}

int sm_count() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[d]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0)
      n = 148;
    g_sms[d] = n;
  }
  return g_sms[d];
}

// Shape rules shared by every op: "What determines your tensor parallel
// degree" requires H % t == 0 (and the FFN width divisible by t); the
// library provides t in {1, 2, 4, 8} ("doesn't recommend going above 8").
tp_status check_common(const tp_dims* d) {
  if (!d) return TP_ERR_INVALID_ARG;
  if (d->batch < 0 || d->seq < 0 || d->hidden <= 0 || d->t <= 0) return TP_ERR_INVALID_ARG;
  if (!supported_t(d->t)) return TP_ERR_UNSUPPORTED;
  // Row counts and tensor-map coordinates are 32-bit.
  if ((long long)d->batch * d->seq > 0x7FFFFFFFLL) return TP_ERR_UNSUPPORTED;
  if (d->hidden % d->t) return TP_ERR_INVALID_ARG;
  if (d->hidden % 8) return TP_ERR_MISALIGNED;
  return TP_OK;
}

tp_status check_mlp(const tp_dims* d) {
  tp_status s = check_common(d);
  if (s != TP_OK) return s;
  if (d->ffn <= 0 || d->ffn % d->t) return TP_ERR_INVALID_ARG;
  if ((d->ffn / d->t) % 8) return TP_ERR_MISALIGNED;
  return TP_OK;
}

tp_status check_attn(const tp_dims* d) {
  tp_status s = check_common(d);
  if (s != TP_OK) return s;
  if (d->heads <= 0 || d->head_dim <= 0) return TP_ERR_INVALID_ARG;
  if ((long long)d->heads * d->head_dim != d->hidden) return TP_ERR_INVALID_ARG;
  if (d->heads % d->t) return TP_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return TP_ERR_UNSUPPORTED;
  if (d->causal != 0 && d->causal != 1) return TP_ERR_INVALID_ARG;
  return TP_OK;
}

tp_status check_layer(const tp_dims* d) {
  tp_status s = check_mlp(d);
  if (s != TP_OK) return s;
  s = check_attn(d);
  if (s != TP_OK) return s;
  if (!(d->ln_eps > 0.f)) return TP_ERR_INVALID_ARG;
  if (d->hidden > 8192) return TP_ERR_UNSUPPORTED;   // LayerNorm register tiling
  return TP_OK;
}

namespace {

using bf16p = const uint16_t*;

struct Sizes {
  long long B, S, T, D, F, H, dh, t, Ft, Dt;
};

Sizes sizes_of(const tp_dims& d) {
  Sizes s{};
  s.B = d.batch;
  s.S = d.seq;
  s.T = (long long)d.batch * d.seq;
  s.D = d.hidden;
  s.F = d.ffn;
  s.H = d.heads;
  s.dh = d.head_dim;
  s.t = d.t;
  s.Ft = d.t > 0 ? d.ffn / d.t : 0;
  s.Dt = d.t > 0 ? d.hidden / d.t : 0;
  return s;
}

OperandDesc op(const void* p, bool mn, int src, long long inner, long long outer,
               long long shards, long long ld, long long shard_stride, bool f16 = false) {
  return OperandDesc{p, mn, f16, src, inner, outer, shards, ld, shard_stride};
}

size_t colsum_scratch_floats_max(long long T, std::initializer_list<std::pair<long long, long long>> sc) {
  size_t m = 0;
  for (auto& p : sc) {
    const size_t f = colsum_partial_floats(p.first, T, p.second);
    if (f > m) m = f;
  }
  return m;
}

// ------------------------------------------------------------------ MLP
tp_status mlp_fwd_impl(const Sizes& z, bf16p x, bf16p w1, bf16p b1, bf16p w2, bf16p b2,
                       bf16p resid, uint16_t* y, uint16_t* a_save, uint16_t* h_save,
                       cudaStream_t st) {
  if (z.T == 0) return TP_OK;
  GemmProblem g1{};
  g1.m_shards = 1; g1.n_shards = (int)z.t; g1.Mt = (int)z.T; g1.Nt = (int)z.Ft;
  g1.k_shards = 1; g1.Kt = (int)z.D;
  g1.a = op(x, false, SHARD_NONE, z.D, z.T, 1, z.D, 0);
  g1.b = op(w1, true, SHARD_MN, z.Ft, z.D, z.t, z.Ft, z.D * z.Ft);
  g1.epi = EPI_BIAS_GELU; g1.c = a_save; g1.c2 = h_save; g1.bias = b1;
  g1.c_ms = 0; g1.c_ns = z.T * z.Ft; g1.ldc = z.Ft;
  tp_status s = launch_gemm(g1, st);
  if (s != TP_OK || y == nullptr) return s;   // y == nullptr: A and H only (recomputation)

  GemmProblem g2{};
  g2.m_shards = 1; g2.n_shards = 1; g2.Mt = (int)z.T; g2.Nt = (int)z.D;
  g2.k_shards = (int)z.t; g2.Kt = (int)z.Ft;
  g2.a = op(h_save, false, SHARD_K, z.Ft, z.T, z.t, z.Ft, z.T * z.Ft);
  g2.b = op(w2, true, SHARD_K, z.D, z.Ft, z.t, z.D, z.Ft * z.D);
  g2.epi = EPI_LINEAR; g2.c = y; g2.bias = b2; g2.aux = resid;
  g2.c_ms = 0; g2.c_ns = 0; g2.ldc = z.D;
  return launch_gemm(g2, st);
}

// Column-sum partial rows of dA that the GeLU' product writes for db1: one per 32 rows.
long long db1_groups(const Sizes& z) { return (z.T + 31) / 32; }

size_t mlp_bwd_ws(const Sizes& z) {
  Carver c(nullptr);
  c.take<uint16_t>((size_t)(z.T * z.F));
  c.take<float>(colsum_scratch_floats_max(z.T, {{1, z.D}}));
  c.take<float>((size_t)(db1_groups(z) * z.F));
  return align_up(c.off, 256);
}

tp_status mlp_bwd_impl(const Sizes& z, bf16p x, bf16p w1, bf16p w2, bf16p a_save, bf16p h_save,
                       bf16p dy, bf16p dres, uint16_t* dx, uint16_t* dw1, uint16_t* dw2,
                       uint16_t* db1, uint16_t* db2, void* ws, cudaStream_t st,
                       const float* dres32 = nullptr, float* dx32 = nullptr) {
  if (z.T == 0) {
    // Sums over zero tokens: all parameter gradients are zero.
    cudaMemsetAsync(dw1, 0, (size_t)(z.D * z.F) * 2, st);
    cudaMemsetAsync(dw2, 0, (size_t)(z.D * z.F) * 2, st);
    if (db1) cudaMemsetAsync(db1, 0, (size_t)z.F * 2, st);
    if (db2) cudaMemsetAsync(db2, 0, (size_t)z.D * 2, st);
    return cuda_status(cudaGetLastError());
  }
  Carver c(ws);
  uint16_t* da = c.take<uint16_t>((size_t)(z.T * z.F));
  float* part = c.take<float>(colsum_scratch_floats_max(z.T, {{1, z.D}}));
  float* dapart = c.take<float>((size_t)(db1_groups(z) * z.F));

  // dA_i = (dY W2_i^T) * GeLU'(A_i): B = W2_i read as [n = Ft][k = D], K-major.
  // db1 = column sums of dA: the epilogue writes one partial row per 32 rows.
  GemmProblem g4{};
  g4.m_shards = 1; g4.n_shards = (int)z.t; g4.Mt = (int)z.T; g4.Nt = (int)z.Ft;
  g4.k_shards = 1; g4.Kt = (int)z.D;
  g4.a = op(dy, false, SHARD_NONE, z.D, z.T, 1, z.D, 0);
  g4.b = op(w2, false, SHARD_MN, z.D, z.Ft, z.t, z.D, z.Ft * z.D);
  g4.epi = EPI_DGELU; g4.c = da; g4.aux = a_save;
  g4.c_ms = 0; g4.c_ns = z.T * z.Ft; g4.ldc = z.Ft;
  if (db1) g4.colpart = dapart;
  tp_status s = launch_gemm(g4, st);
  if (s != TP_OK) return s;
  if (db1 && (s = launch_colsum_reduce(dapart, db1_groups(z), z.F, db1, st)) != TP_OK) return s;

  // dW2_i = H_i^T dY: A = H_i^T (M-major), M shards.
  GemmProblem g5{};
  g5.m_shards = (int)z.t; g5.n_shards = 1; g5.Mt = (int)z.Ft; g5.Nt = (int)z.D;
  g5.k_shards = 1; g5.Kt = (int)z.T;
  g5.a = op(h_save, true, SHARD_MN, z.Ft, z.T, z.t, z.Ft, z.T * z.Ft);
  g5.b = op(dy, true, SHARD_NONE, z.D, z.T, 1, z.D, 0);
  g5.epi = EPI_LINEAR; g5.c = dw2;
  g5.c_ms = z.Ft * z.D; g5.c_ns = 0; g5.ldc = z.D;
  if ((s = launch_gemm(g5, st)) != TP_OK) return s;

  // dW1_i = x^T dA_i: N shards.
  GemmProblem g6{};
  g6.m_shards = 1; g6.n_shards = (int)z.t; g6.Mt = (int)z.D; g6.Nt = (int)z.Ft;
  g6.k_shards = 1; g6.Kt = (int)z.T;
  g6.a = op(x, true, SHARD_NONE, z.D, z.T, 1, z.D, 0);
  g6.b = op(da, true, SHARD_MN, z.Ft, z.T, z.t, z.Ft, z.T * z.Ft);
  g6.epi = EPI_LINEAR; g6.c = dw1;
  g6.c_ms = 0; g6.c_ns = z.D * z.Ft; g6.ldc = z.Ft;
  if ((s = launch_gemm(g6, st)) != TP_OK) return s;

  // dX = sum_i dA_i W1_i^T (+ dres): the backward shard reduction, K shards.
  GemmProblem g7{};
  g7.m_shards = 1; g7.n_shards = 1; g7.Mt = (int)z.T; g7.Nt = (int)z.D;
  g7.k_shards = (int)z.t; g7.Kt = (int)z.Ft;
  g7.a = op(da, false, SHARD_K, z.Ft, z.T, z.t, z.Ft, z.T * z.Ft);
  g7.b = op(w1, false, SHARD_K, z.Ft, z.D, z.t, z.Ft, z.D * z.Ft);
  g7.epi = EPI_LINEAR; g7.c = dx; g7.aux = dres;
  if (dres32) { g7.aux = dres32; g7.aux_f32 = true; }
  if (dx32) { g7.c = dx32; g7.out_f32 = true; }
  g7.c_ms = 0; g7.c_ns = 0; g7.ldc = z.D;
  if ((s = launch_gemm(g7, st)) != TP_OK) return s;

  if (db2 && (s = launch_colsum_stacked(dy, 1, z.T, z.D, db2, part, st)) != TP_OK) return s;
  return TP_OK;
}

// ------------------------------------------------------------------ attention
// The attention sublayer runs on fp16 operands internally (see attention.cu
// for why): its input x16 and the fp16 copy of Wqkv are prepared by the
// caller of these helpers; qkv is stored fp16, O bf16.
tp_status attn_fwd_impl(const Sizes& z, int causal, bf16p x16, bf16p wqkv16, bf16p bqkv,
                        bf16p wout, bf16p bout, bf16p resid, uint16_t* y, uint16_t* qkv,
                        uint16_t* o, float* lse, cudaStream_t st) {
  if (z.T == 0) return TP_OK;
  const long long w3 = 3 * z.Dt;
  GemmProblem g1{};
  g1.m_shards = 1; g1.n_shards = (int)z.t; g1.Mt = (int)z.T; g1.Nt = (int)w3;
  g1.k_shards = 1; g1.Kt = (int)z.D;
  g1.a = op(x16, false, SHARD_NONE, z.D, z.T, 1, z.D, 0, true);
  g1.b = op(wqkv16, true, SHARD_MN, w3, z.D, z.t, w3, z.D * w3, true);
  g1.epi = EPI_LINEAR; g1.c = qkv; g1.bias = bqkv; g1.out_f16 = true;
  g1.c_ms = 0; g1.c_ns = z.T * w3; g1.ldc = w3;
  tp_status s = launch_gemm(g1, st);
  if (s != TP_OK) return s;

  s = launch_attn_fwd(qkv, o, lse, (int)z.B, (int)z.S, (int)z.H, (int)z.dh, (int)z.t, causal, st);
  if (s != TP_OK) return s;

  GemmProblem g2{};
  g2.m_shards = 1; g2.n_shards = 1; g2.Mt = (int)z.T; g2.Nt = (int)z.D;
  g2.k_shards = (int)z.t; g2.Kt = (int)z.Dt;
  g2.a = op(o, false, SHARD_K, z.Dt, z.T, z.t, z.Dt, z.T * z.Dt);
  g2.b = op(wout, true, SHARD_K, z.D, z.Dt, z.t, z.D, z.Dt * z.D);
  g2.epi = EPI_LINEAR; g2.c = y; g2.bias = bout; g2.aux = resid;
  g2.c_ms = 0; g2.c_ns = 0; g2.ldc = z.D;
  return launch_gemm(g2, st);
}

// Workspace of attn_bwd_impl: dO (fp16), dqkv (fp16), attention scratch, colsum
// partials of dy (dbout) and the dqkv column partials the attention kernels write (dbqkv).
size_t attn_bwd_core_ws(const Sizes& z) {
  Carver c(nullptr);
  c.take<uint16_t>((size_t)(z.T * z.D));
  c.take<uint16_t>((size_t)(z.T * 3 * z.D));
  c.take<uint8_t>(attn_bwd_scratch_bytes((int)z.B, (int)z.S, (int)z.H, (int)z.dh));
  c.take<float>(colsum_scratch_floats_max(z.T, {{1, z.D}}));
  c.take<float>((size_t)(attn_colpart_rows(z.B, z.S) * 3 * z.D));
  return align_up(c.off, 256);
}

tp_status attn_bwd_impl(const Sizes& z, int causal, bf16p x16, bf16p wqkv16, bf16p wout,
                        bf16p qkv, bf16p o, const float* lse, bf16p dy, bf16p dres, uint16_t* dx,
                        uint16_t* dwqkv, uint16_t* dbqkv, uint16_t* dwout, uint16_t* dbout,
                        void* ws, cudaStream_t st, const float* dres32 = nullptr) {
  const long long w3 = 3 * z.Dt;
  if (z.T == 0) {
    cudaMemsetAsync(dwqkv, 0, (size_t)(z.D * 3 * z.D) * 2, st);
    cudaMemsetAsync(dwout, 0, (size_t)(z.D * z.D) * 2, st);
    if (dbqkv) cudaMemsetAsync(dbqkv, 0, (size_t)(3 * z.D) * 2, st);
    if (dbout) cudaMemsetAsync(dbout, 0, (size_t)z.D * 2, st);
    return cuda_status(cudaGetLastError());
  }
  Carver c(ws);
  uint16_t* dout = c.take<uint16_t>((size_t)(z.T * z.D));
  uint16_t* dqkv = c.take<uint16_t>((size_t)(z.T * 3 * z.D));
  void* scratch = c.take<uint8_t>(attn_bwd_scratch_bytes((int)z.B, (int)z.S, (int)z.H, (int)z.dh));
  float* part = c.take<float>(colsum_scratch_floats_max(z.T, {{1, z.D}}));
  float* qkvpart = c.take<float>((size_t)(attn_colpart_rows(z.B, z.S) * 3 * z.D));

  // dO_i = dY Wout_i^T: B = Wout_i read as [n = Dt][k = D], K-major, N shards; fp16 out.
  GemmProblem g1{};
  g1.m_shards = 1; g1.n_shards = (int)z.t; g1.Mt = (int)z.T; g1.Nt = (int)z.Dt;
  g1.k_shards = 1; g1.Kt = (int)z.D;
  g1.a = op(dy, false, SHARD_NONE, z.D, z.T, 1, z.D, 0);
  g1.b = op(wout, false, SHARD_MN, z.D, z.Dt, z.t, z.D, z.Dt * z.D);
  g1.epi = EPI_LINEAR; g1.c = dout; g1.out_f16 = true;
  g1.c_ms = 0; g1.c_ns = z.T * z.Dt; g1.ldc = z.Dt;
  tp_status s = launch_gemm(g1, st);
  if (s != TP_OK) return s;

  // dWout_i = O_i^T dY, M shards (launched below together with dWqkv: its
  // 16 x 16 tiles alone leave the last round of clusters half empty).
  GemmProblem g2{};
  g2.m_shards = (int)z.t; g2.n_shards = 1; g2.Mt = (int)z.Dt; g2.Nt = (int)z.D;
  g2.k_shards = 1; g2.Kt = (int)z.T;
  g2.a = op(o, true, SHARD_MN, z.Dt, z.T, z.t, z.Dt, z.T * z.Dt);
  g2.b = op(dy, true, SHARD_NONE, z.D, z.T, 1, z.D, 0);
  g2.epi = EPI_LINEAR; g2.c = dwout;
  g2.c_ms = z.Dt * z.D; g2.c_ns = 0; g2.ldc = z.D;

  // dbqkv = column sums of dqkv: the attention kernels' epilogues write partials.
  s = launch_attn_bwd(qkv, o, lse, dout, dqkv, (int)z.B, (int)z.S, (int)z.H, (int)z.dh, (int)z.t,
                      causal, scratch, st, dbqkv ? qkvpart : nullptr);
  if (s != TP_OK) return s;
  if (dbqkv && (s = launch_colsum_reduce(qkvpart, attn_colpart_rows(z.B, z.S), 3 * z.D, dbqkv,
                                         st)) != TP_OK)
    return s;

  // dWqkv_i = x^T dqkv_i, N shards (fp16 operands).
  GemmProblem g3{};
  g3.m_shards = 1; g3.n_shards = (int)z.t; g3.Mt = (int)z.D; g3.Nt = (int)w3;
  g3.k_shards = 1; g3.Kt = (int)z.T;
  g3.a = op(x16, true, SHARD_NONE, z.D, z.T, 1, z.D, 0, true);
  g3.b = op(dqkv, true, SHARD_MN, w3, z.T, z.t, w3, z.T * w3, true);
  g3.epi = EPI_LINEAR; g3.c = dwqkv;
  g3.c_ms = 0; g3.c_ns = z.D * w3; g3.ldc = w3;
  if ((s = launch_gemm2(g2, g3, st)) != TP_OK) return s;

  // dX = sum_i dqkv_i Wqkv_i^T (+ dres): the backward shard reduction (fp16 operands).
  GemmProblem g4{};
  g4.m_shards = 1; g4.n_shards = 1; g4.Mt = (int)z.T; g4.Nt = (int)z.D;
  g4.k_shards = (int)z.t; g4.Kt = (int)w3;
  g4.a = op(dqkv, false, SHARD_K, w3, z.T, z.t, w3, z.T * w3, true);
  g4.b = op(wqkv16, false, SHARD_K, w3, z.D, z.t, w3, z.D * w3, true);
  g4.epi = EPI_LINEAR; g4.c = dx; g4.aux = dres;
  if (dres32) { g4.aux = dres32; g4.aux_f32 = true; }
  g4.c_ms = 0; g4.c_ns = 0; g4.ldc = z.D;
  if ((s = launch_gemm(g4, st)) != TP_OK) return s;

  if (dbout && (s = launch_colsum_stacked(dy, 1, z.T, z.D, dbout, part, st)) != TP_OK) return s;
  return TP_OK;
}

// Standalone attention: fp16 copies of x and Wqkv, then the core workspace.
size_t attn_fwd_ws(const Sizes& z) {
  Carver c(nullptr);
  c.take<uint16_t>((size_t)(z.T * z.D));
  c.take<uint16_t>((size_t)(z.D * 3 * z.D));
  return align_up(c.off, 256);
}

size_t attn_bwd_ws(const Sizes& z) {
  return attn_fwd_ws(z) + attn_bwd_core_ws(z);
}

size_t layer_fwd_ws(const Sizes& z) {
  return align_up((size_t)(z.D * 3 * z.D) * 2, 256);   // fp16 copy of Wqkv
}

size_t layer_bwd_ws(const Sizes& z) {
  Carver c(nullptr);
  c.take<uint16_t>((size_t)(z.D * 3 * z.D));   // fp16 copy of Wqkv
  c.take<uint16_t>((size_t)(z.T * z.D));       // du
  c.take<uint16_t>((size_t)(z.T * z.D));       // dh
  c.take<float>(layernorm_bwd_partial_floats(z.T, (int)z.D, 3));
  const size_t sub = mlp_bwd_ws(z) > attn_bwd_core_ws(z) ? mlp_bwd_ws(z) : attn_bwd_core_ws(z);
  c.take<uint8_t>(sub);
  return align_up(c.off, 256);
}

// The pre-LN layer's saved activations carved out of a workspace (the
// recomputation entry points keep them there instead of in caller buffers).
tp_layer_acts carve_layer_acts(Carver& c, const Sizes& z) {
  tp_layer_acts a{};
  a.u1 = c.take<uint16_t>((size_t)(z.T * z.D));
  a.mean1 = c.take<float>((size_t)z.T);
  a.rstd1 = c.take<float>((size_t)z.T);
  a.qkv = c.take<uint16_t>((size_t)(z.T * 3 * z.D));
  a.o = c.take<uint16_t>((size_t)(z.T * z.D));
  a.lse = c.take<float>((size_t)(z.B * z.H * z.S));
  a.h = c.take<uint16_t>((size_t)(z.T * z.D));
  a.u2 = c.take<uint16_t>((size_t)(z.T * z.D));
  a.mean2 = c.take<float>((size_t)z.T);
  a.rstd2 = c.take<float>((size_t)z.T);
  a.a = c.take<uint16_t>((size_t)(z.T * z.F));
  a.hact = c.take<uint16_t>((size_t)(z.T * z.F));
  return a;
}

size_t layer_acts_ws(const Sizes& z) {
  Carver c(nullptr);
  carve_layer_acts(c, z);
  return align_up(c.off, 256);
}

size_t layer_fwd_nosave_ws(const Sizes& z) { return layer_fwd_ws(z) + layer_acts_ws(z); }
size_t layer_bwd_recompute_ws(const Sizes& z) { return layer_acts_ws(z) + layer_bwd_ws(z); }

// Post-LN layer workspaces: fp16 copies of x and Wqkv (forward and backward),
// plus the gradient chain, LayerNorm partials and the sublayer workspace
// (backward).  The chain dz2 -> dh -> dz1 passes through two LayerNorm
// Jacobians and two residual additions; rounding each link to bf16 compounds
// to about twice the per-element error of the pre-LN layer, so the links are
// carried in fp32 and only the GEMM operands are bf16: one bf16 buffer (dz2,
// then dz1), one fp32 buffer (dz2, then dz1) and fp32 dh.
size_t postln_fwd_ws(const Sizes& z) { return attn_fwd_ws(z); }

size_t postln_bwd_ws(const Sizes& z) {
  Carver c(nullptr);
  c.take<uint8_t>(attn_fwd_ws(z));
  c.take<uint16_t>((size_t)(z.T * z.D));
  c.take<float>((size_t)(z.T * z.D));
  c.take<float>((size_t)(z.T * z.D));
  c.take<float>(layernorm_bwd_partial_floats(z.T, (int)z.D));
  const size_t sub = mlp_bwd_ws(z) > attn_bwd_core_ws(z) ? mlp_bwd_ws(z) : attn_bwd_core_ws(z);
  c.take<uint8_t>(sub);
  return align_up(c.off, 256);
}

}  // namespace
}  // namespace tp

using namespace tp;

extern "C" {

const char* tp_version(void) { return "tplayer-b200 0.1 (sm_100a)"; }

const char* tp_status_string(tp_status s) {
  switch (s) {
    case TP_OK: return "TP_OK";
    case TP_ERR_INVALID_ARG: return "TP_ERR_INVALID_ARG";
    case TP_ERR_UNSUPPORTED: return "TP_ERR_UNSUPPORTED";
    case TP_ERR_MISALIGNED: return "TP_ERR_MISALIGNED";
    case TP_ERR_WORKSPACE: return "TP_ERR_WORKSPACE";
    case TP_ERR_CUDA: return "TP_ERR_CUDA";
    case TP_ERR_TIMEOUT: return "TP_ERR_TIMEOUT";
    case TP_ERR_RANGE: return "TP_ERR_RANGE";
  }
  return "TP_ERR_UNKNOWN";
}

size_t tp_attn_set_ds_limit(size_t max_bytes) { return attn_set_dst_limit(max_bytes); }

size_t tp_workspace_size(int op_, const tp_dims* d) {
  DstLimitPin pin;   // one dS^T limit for the whole call
  switch (op_) {
    case TP_OP_MLP_FWD: return 0;
    case TP_OP_ATTN_FWD: return check_attn(d) == TP_OK ? attn_fwd_ws(sizes_of(*d)) : 0;
    case TP_OP_LAYER_FWD: return check_layer(d) == TP_OK ? layer_fwd_ws(sizes_of(*d)) : 0;
    case TP_OP_MLP_BWD: return check_mlp(d) == TP_OK ? mlp_bwd_ws(sizes_of(*d)) : 0;
    case TP_OP_ATTN_BWD: return check_attn(d) == TP_OK ? attn_bwd_ws(sizes_of(*d)) : 0;
    case TP_OP_LAYER_BWD: return check_layer(d) == TP_OK ? layer_bwd_ws(sizes_of(*d)) : 0;
    case TP_OP_POSTLN_FWD: return check_layer(d) == TP_OK ? postln_fwd_ws(sizes_of(*d)) : 0;
    case TP_OP_POSTLN_BWD: return check_layer(d) == TP_OK ? postln_bwd_ws(sizes_of(*d)) : 0;
    case TP_OP_LAYER_FWD_NOSAVE:
      return check_layer(d) == TP_OK ? layer_fwd_nosave_ws(sizes_of(*d)) : 0;
    case TP_OP_LAYER_BWD_RECOMPUTE:
      return check_layer(d) == TP_OK ? layer_bwd_recompute_ws(sizes_of(*d)) : 0;
  }
  return 0;
}

tp_status tp_check_error(unsigned int* code) {
  if (cudaDeviceSynchronize() != cudaSuccess) return TP_ERR_CUDA;
  unsigned int* p = error_word();
  if (!p) return TP_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return TP_ERR_CUDA;
  if (v != 0) {
    const unsigned int zero = 0;
    cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice);
  }
  if (code) *code = v;
  if (v == 0) return TP_OK;
  return (v & 0xF00u) == 0x300u ? TP_ERR_RANGE : TP_ERR_TIMEOUT;
}

// ------------------------------------------------------------------ layout
static tp_status check_layout(const void* a, const void* b, int rows, int cols, int t) {
  if (!a || !b || rows < 0 || cols < 0) return TP_ERR_INVALID_ARG;
  if (!supported_t(t)) return TP_ERR_UNSUPPORTED;
  if (cols % t) return TP_ERR_INVALID_ARG;
  return TP_OK;
}

tp_status tp_shard_cols(const tp_bf16* w, int rows, int cols, int t, tp_bf16* out, tp_stream s) {
  tp_status st = check_layout(w, out, rows, cols, t);
  if (st != TP_OK) return st;
  return launch_shard_cols(w, rows, cols, t, out, false, (cudaStream_t)s);
}

tp_status tp_unshard_cols(const tp_bf16* p, int rows, int cols, int t, tp_bf16* w, tp_stream s) {
  tp_status st = check_layout(p, w, rows, cols, t);
  if (st != TP_OK) return st;
  return launch_shard_cols(p, rows, cols, t, w, true, (cudaStream_t)s);
}

tp_status tp_shard_rows(const tp_bf16* w, int rows, int cols, int t, tp_bf16* out, tp_stream s) {
  if (!w || !out || rows < 0 || cols < 0) return TP_ERR_INVALID_ARG;
  if (!supported_t(t)) return TP_ERR_UNSUPPORTED;
  if (rows % t) return TP_ERR_INVALID_ARG;
  return launch_copy(w, (size_t)rows * cols, out, (cudaStream_t)s);
}

tp_status tp_unshard_rows(const tp_bf16* p, int rows, int cols, int t, tp_bf16* w, tp_stream s) {
  return tp_shard_rows(p, rows, cols, t, w, s);
}

static tp_status check_qkv(const void* a, const void* b, int rows, int hidden, int heads, int t) {
  if (!a || !b || rows < 0 || hidden <= 0 || heads <= 0) return TP_ERR_INVALID_ARG;
  if (!supported_t(t)) return TP_ERR_UNSUPPORTED;
  if (heads % t || hidden % heads) return TP_ERR_INVALID_ARG;
  return TP_OK;
}

tp_status tp_shard_qkv_heads(const tp_bf16* w, int rows, int hidden, int heads, int t, tp_bf16* out,
                             tp_stream s) {
  tp_status st = check_qkv(w, out, rows, hidden, heads, t);
  if (st != TP_OK) return st;
  return launch_shard_qkv(w, rows, hidden, t, out, false, (cudaStream_t)s);
}

tp_status tp_unshard_qkv_heads(const tp_bf16* p, int rows, int hidden, int heads, int t,
                               tp_bf16* w, tp_stream s) {
  tp_status st = check_qkv(p, w, rows, hidden, heads, t);
  if (st != TP_OK) return st;
  return launch_shard_qkv(p, rows, hidden, t, w, true, (cudaStream_t)s);
}

// ------------------------------------------------------------------ MLP
tp_status tp_mlp_fwd(const tp_dims* dims, const tp_bf16* x, const tp_bf16* w1, const tp_bf16* b1,
                     const tp_bf16* w2, const tp_bf16* b2, const tp_bf16* resid, tp_bf16* y,
                     tp_bf16* a_save, tp_bf16* h_save, void* ws, size_t ws_bytes, tp_stream s) {
  (void)ws; (void)ws_bytes;
  tp_status st = check_mlp(dims);
  if (st != TP_OK) return st;
  const bool tok = (long long)dims->batch * dims->seq > 0;   // activations may be NULL when T == 0
  if (!all_set(w1, w2) || (tok && !all_set(x, y, a_save, h_save))) return TP_ERR_INVALID_ARG;
  if (!all_aligned(x, w1, b1, w2, b2, resid, y, a_save, h_save)) return TP_ERR_MISALIGNED;
  return mlp_fwd_impl(sizes_of(*dims), x, w1, b1, w2, b2, resid, y, a_save, h_save,
                      (cudaStream_t)s);
}

tp_status tp_mlp_bwd(const tp_dims* dims, const tp_bf16* x, const tp_bf16* w1, const tp_bf16* w2,
                     const tp_bf16* a_save, const tp_bf16* h_save, const tp_bf16* dy,
                     const tp_bf16* dres, tp_bf16* dx, tp_bf16* dw1, tp_bf16* dw2, tp_bf16* db1,
                     tp_bf16* db2, void* ws, size_t ws_bytes, tp_stream s) {
  tp_status st = check_mlp(dims);
  if (st != TP_OK) return st;
  const bool tok = (long long)dims->batch * dims->seq > 0;
  if (!all_set(w1, w2, dw1, dw2) || (tok && !all_set(x, a_save, h_save, dy, dx)))
    return TP_ERR_INVALID_ARG;
  if (!all_aligned(x, w1, w2, a_save, h_save, dy, dres, dx, dw1, dw2, db1, db2))
    return TP_ERR_MISALIGNED;
  const Sizes z = sizes_of(*dims);
  if ((st = check_ws(ws, ws_bytes, z.T ? mlp_bwd_ws(z) : 0)) != TP_OK) return st;
  return mlp_bwd_impl(z, x, w1, w2, a_save, h_save, dy, dres, dx, dw1, dw2, db1, db2, ws,
                      (cudaStream_t)s);
}

// ------------------------------------------------------------------ attention
tp_status tp_attn_fwd(const tp_dims* dims, const tp_bf16* x, const tp_bf16* wqkv,
                      const tp_bf16* bqkv, const tp_bf16* wout, const tp_bf16* bout,
                      const tp_bf16* resid, tp_bf16* y, tp_f16* qkv_save, tp_bf16* o_save,
                      float* lse_save, void* ws, size_t ws_bytes, tp_stream s) {
  tp_status st = check_attn(dims);
  if (st != TP_OK) return st;
  const bool tok = (long long)dims->batch * dims->seq > 0;
  if (!all_set(wqkv, wout) || (tok && !all_set(x, y, qkv_save, o_save, lse_save)))
    return TP_ERR_INVALID_ARG;
  if (!all_aligned(x, wqkv, bqkv, wout, bout, resid, y, qkv_save, o_save, lse_save))
    return TP_ERR_MISALIGNED;
  const Sizes z = sizes_of(*dims);
  if (z.T == 0) return TP_OK;
  if ((st = check_ws(ws, ws_bytes, attn_fwd_ws(z))) != TP_OK) return st;
  cudaStream_t cs = (cudaStream_t)s;
  Carver c(ws);
  uint16_t* x16 = c.take<uint16_t>((size_t)(z.T * z.D));
  uint16_t* w16 = c.take<uint16_t>((size_t)(z.D * 3 * z.D));
  if ((st = launch_cast_f16(x, (size_t)(z.T * z.D), x16, cs)) != TP_OK) return st;
  if ((st = launch_cast_f16(wqkv, (size_t)(z.D * 3 * z.D), w16, cs)) != TP_OK) return st;
  return attn_fwd_impl(z, dims->causal, x16, w16, bqkv, wout, bout, resid, y, qkv_save, o_save,
                       lse_save, cs);
}

tp_status tp_attn_bwd(const tp_dims* dims, const tp_bf16* x, const tp_bf16* wqkv,
                      const tp_bf16* wout, const tp_f16* qkv_save, const tp_bf16* o_save,
                      const float* lse_save, const tp_bf16* dy, const tp_bf16* dres, tp_bf16* dx,
                      tp_bf16* dwqkv, tp_bf16* dbqkv, tp_bf16* dwout, tp_bf16* dbout, void* ws,
                      size_t ws_bytes, tp_stream s) {
  DstLimitPin pin;   // one dS^T limit for the whole call
  tp_status st = check_attn(dims);
  if (st != TP_OK) return st;
  const bool tok = (long long)dims->batch * dims->seq > 0;
  if (!all_set(wqkv, wout, dwqkv, dwout) ||
      (tok && !all_set(x, qkv_save, o_save, lse_save, dy, dx)))
    return TP_ERR_INVALID_ARG;
  if (!all_aligned(x, wqkv, wout, qkv_save, o_save, lse_save, dy, dres, dx, dwqkv, dbqkv, dwout,
                   dbout))
    return TP_ERR_MISALIGNED;
  const Sizes z = sizes_of(*dims);
  if ((st = check_ws(ws, ws_bytes, z.T ? attn_bwd_ws(z) : 0)) != TP_OK) return st;
  cudaStream_t cs = (cudaStream_t)s;
  if (z.T == 0)
    return attn_bwd_impl(z, dims->causal, nullptr, nullptr, wout, nullptr, nullptr, nullptr,
                         nullptr, nullptr, nullptr, dwqkv, dbqkv, dwout, dbout, nullptr, cs);
  Carver c(ws);
  uint16_t* x16 = c.take<uint16_t>((size_t)(z.T * z.D));
  uint16_t* w16 = c.take<uint16_t>((size_t)(z.D * 3 * z.D));
  void* core = c.take<uint8_t>(attn_bwd_core_ws(z));
  if ((st = launch_cast_f16(x, (size_t)(z.T * z.D), x16, cs)) != TP_OK) return st;
  if ((st = launch_cast_f16(wqkv, (size_t)(z.D * 3 * z.D), w16, cs)) != TP_OK) return st;
  return attn_bwd_impl(z, dims->causal, x16, w16, wout, qkv_save, o_save, lse_save, dy, dres, dx,
                       dwqkv, dbqkv, dwout, dbout, core, cs);
}

// ------------------------------------------------------------------ LayerNorm
tp_status tp_layernorm_fwd(const tp_bf16* x, const tp_bf16* gamma, const tp_bf16* beta, int rows,
                           int D, float eps, tp_bf16* y, float* mean, float* rstd, tp_stream s) {
  if (!all_set(x, gamma, beta, y, mean, rstd) || rows < 0 || D <= 0 || !(eps > 0.f))
    return TP_ERR_INVALID_ARG;
  if (D > 8192) return TP_ERR_UNSUPPORTED;
  if (D % 8 || !all_aligned(x, gamma, beta, y)) return TP_ERR_MISALIGNED;
  return launch_layernorm_fwd(x, gamma, beta, rows, D, eps, y, mean, rstd, (cudaStream_t)s);
}

tp_status tp_layernorm_fwd_f16(const tp_bf16* x, const tp_bf16* gamma, const tp_bf16* beta,
                               int rows, int D, float eps, tp_f16* y, float* mean, float* rstd,
                               tp_stream s) {
  if (!all_set(x, gamma, beta, y, mean, rstd) || rows < 0 || D <= 0 || !(eps > 0.f))
    return TP_ERR_INVALID_ARG;
  if (D > 8192) return TP_ERR_UNSUPPORTED;
  if (D % 8 || !all_aligned(x, gamma, beta, y)) return TP_ERR_MISALIGNED;
  return launch_layernorm_fwd(x, gamma, beta, rows, D, eps, y, mean, rstd, (cudaStream_t)s, true);
}

size_t tp_layernorm_bwd_workspace_size(int rows, int D) {
  if (rows < 0 || D <= 0) return 0;
  return align_up(layernorm_bwd_partial_floats(rows, D) * sizeof(float), 256);
}

tp_status tp_layernorm_bwd(const tp_bf16* dy, const tp_bf16* x, const tp_bf16* gamma,
                           const float* mean, const float* rstd, const tp_bf16* dres, int rows,
                           int D, tp_bf16* dx, tp_bf16* dgamma, tp_bf16* dbeta, void* ws,
                           size_t ws_bytes, tp_stream s) {
  if (!all_set(dy, x, gamma, mean, rstd, dx) || rows < 0 || D <= 0) return TP_ERR_INVALID_ARG;
  if (D > 8192) return TP_ERR_UNSUPPORTED;
  if (D % 8 || !all_aligned(dy, x, gamma, dres, dx)) return TP_ERR_MISALIGNED;
  tp_status st = check_ws(ws, ws_bytes, tp_layernorm_bwd_workspace_size(rows, D));
  if (st != TP_OK) return st;
  return launch_layernorm_bwd(dy, x, gamma, mean, rstd, dres, rows, D, dx, dgamma, dbeta,
                              static_cast<float*>(ws), (cudaStream_t)s);
}

// ------------------------------------------------------------------ pre-LN layer
// Saved activations (and x, y) may be NULL when the layer has zero tokens.
static bool has_tokens(const tp_dims* d) { return (long long)d->batch * d->seq > 0; }

static tp_status check_layer_ptrs(const tp_layer_params* p, const tp_layer_acts* a, bool tok) {
  if (!p || !a) return TP_ERR_INVALID_ARG;
  if (!all_set(p->ln1_g, p->ln1_b, p->wqkv, p->wout, p->ln2_g, p->ln2_b, p->w1, p->w2))
    return TP_ERR_INVALID_ARG;
  if (tok && !all_set(a->u1, a->mean1, a->rstd1, a->qkv, a->o, a->lse, a->h, a->u2, a->mean2,
                      a->rstd2, a->a, a->hact))
    return TP_ERR_INVALID_ARG;
  if (!all_aligned(p->ln1_g, p->ln1_b, p->wqkv, p->bqkv, p->wout, p->bout, p->ln2_g, p->ln2_b,
                   p->w1, p->b1, p->w2, p->b2))
    return TP_ERR_MISALIGNED;
  if (!all_aligned(a->u1, a->qkv, a->o, a->lse, a->h, a->u2, a->a, a->hact, a->wqkv16))
    return TP_ERR_MISALIGNED;
  return TP_OK;
}

}  // extern "C"

namespace tp {
namespace {

// Pre-LN forward on activations `a`, with the fp16 copy of Wqkv already in
// w16.  y == nullptr leaves out the MLP's second product (recomputation).
tp_status layer_fwd_core(const Sizes& z, const tp_dims* dims, const tp_bf16* x,
                         const tp_layer_params* p, const tp_layer_acts* a, tp_bf16* y,
                         const uint16_t* w16, cudaStream_t cs) {
  tp_status st;
  // LN1 writes u1 in fp16: it only feeds the attention sublayer's fp16 products.
  if ((st = launch_layernorm_fwd(x, p->ln1_g, p->ln1_b, z.T, (int)z.D, dims->ln_eps, a->u1,
                                 a->mean1, a->rstd1, cs, true)) != TP_OK)
    return st;
  if ((st = attn_fwd_impl(z, dims->causal, a->u1, w16, p->bqkv, p->wout, p->bout, x, a->h,
                          a->qkv, a->o, a->lse, cs)) != TP_OK)
    return st;
  if ((st = launch_layernorm_fwd(a->h, p->ln2_g, p->ln2_b, z.T, (int)z.D, dims->ln_eps, a->u2,
                                 a->mean2, a->rstd2, cs)) != TP_OK)
    return st;
  return mlp_fwd_impl(z, a->u2, p->w1, p->b1, p->w2, p->b2, a->h, y, a->a, a->hact, cs);
}

// Records `ev` (a caller's cudaEvent_t, may be NULL) on the stream.
tp_status record_ready(void* ev, cudaStream_t cs) {
  if (ev == nullptr) return TP_OK;
  return cuda_status(cudaEventRecord(static_cast<cudaEvent_t>(ev), cs));
}

// Pre-LN backward; `ws` is laid out as layer_bwd_ws describes.  The fp16 copy
// of Wqkv is the forward's (a->wqkv16) when the caller kept it, otherwise it
// is made here in the workspace's first slice.
tp_status layer_bwd_core(const Sizes& z, const tp_dims* dims, const tp_bf16* x,
                         const tp_layer_params* p, const tp_layer_acts* a, const tp_bf16* dy,
                         tp_bf16* dx, const tp_layer_grads* g, void* ws, cudaStream_t cs,
                         const tp_grad_ready* ready = nullptr) {
  tp_status st;
  Carver c(ws);
  uint16_t* w16 = c.take<uint16_t>((size_t)(z.D * 3 * z.D));
  if (a->wqkv16 != nullptr) {
    w16 = a->wqkv16;
  } else if ((st = launch_cast_f16(p->wqkv, (size_t)(z.D * 3 * z.D), w16, cs)) != TP_OK) {
    return st;
  }
  uint16_t* du = c.take<uint16_t>((size_t)(z.T * z.D));
  uint16_t* dh = c.take<uint16_t>((size_t)(z.T * z.D));
  float* lnp = c.take<float>(layernorm_bwd_partial_floats(z.T, (int)z.D, 3));
  const size_t sub = mlp_bwd_ws(z) > attn_bwd_core_ws(z) ? mlp_bwd_ws(z) : attn_bwd_core_ws(z);
  void* subws = c.take<uint8_t>(sub);

  // y = h + MLP(LN2(h)):  du2 = MLP^T(dy);  dh = dy + LN2^T(du2).  db2 = column
  // sums of dy, which LN2's backward reads as the residual gradient anyway.
  if ((st = mlp_bwd_impl(z, a->u2, p->w1, p->w2, a->a, a->hact, dy, nullptr, du, g->dw1, g->dw2,
                         g->db1, nullptr, subws, cs)) != TP_OK)
    return st;
  if ((st = launch_layernorm_bwd(du, a->h, p->ln2_g, a->mean2, a->rstd2, dy, z.T, (int)z.D, dh,
                                 g->dln2_g, g->dln2_b, lnp, cs, nullptr, g->db2)) != TP_OK)
    return st;
  if (ready && (st = record_ready(ready->mlp, cs)) != TP_OK) return st;
  // h = x + Attn(LN1(x)):  du1 = Attn^T(dh);  dx = dh + LN1^T(du1).  dbout =
  // column sums of dh, read by LN1's backward as its residual gradient.
  if ((st = attn_bwd_impl(z, dims->causal, a->u1, w16, p->wout, a->qkv, a->o, a->lse, dh,
                          nullptr, du, g->dwqkv, g->dbqkv, g->dwout, nullptr, subws, cs)) != TP_OK)
    return st;
  if (ready && (st = record_ready(ready->attn, cs)) != TP_OK) return st;
  if ((st = launch_layernorm_bwd(du, x, p->ln1_g, a->mean1, a->rstd1, dh, z.T, (int)z.D, dx,
                                 g->dln1_g, g->dln1_b, lnp, cs, nullptr, g->dbout)) != TP_OK)
    return st;
  return ready ? record_ready(ready->ln1, cs) : TP_OK;
}

tp_status check_layer_params(const tp_layer_params* p) {
  if (!p) return TP_ERR_INVALID_ARG;
  if (!all_set(p->ln1_g, p->ln1_b, p->wqkv, p->wout, p->ln2_g, p->ln2_b, p->w1, p->w2))
    return TP_ERR_INVALID_ARG;
  if (!all_aligned(p->ln1_g, p->ln1_b, p->wqkv, p->bqkv, p->wout, p->bout, p->ln2_g, p->ln2_b,
                   p->w1, p->b1, p->w2, p->b2))
    return TP_ERR_MISALIGNED;
  return TP_OK;
}

// Activations (x, dy, dx) may be NULL when the layer has zero tokens.
tp_status check_layer_grads(const tp_dims* d, const tp_bf16* x, const tp_bf16* dy,
                            const tp_bf16* dx, const tp_layer_grads* g) {
  const bool tok = (long long)d->batch * d->seq > 0;
  if (!g || (tok && !all_set(x, dy, dx))) return TP_ERR_INVALID_ARG;
  if (!all_set(g->dwqkv, g->dwout, g->dw1, g->dw2)) return TP_ERR_INVALID_ARG;
  if (!all_aligned(x, dy, dx, g->dln1_g, g->dln1_b, g->dwqkv, g->dbqkv, g->dwout, g->dbout,
                   g->dln2_g, g->dln2_b, g->dw1, g->db1, g->dw2, g->db2))
    return TP_ERR_MISALIGNED;
  return TP_OK;
}

// Gradients of a layer over zero tokens: every parameter gradient is zero.
tp_status layer_bwd_empty(const Sizes& z, int causal, const tp_layer_grads* g, cudaStream_t cs) {
  mlp_bwd_impl(z, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, g->dw1,
               g->dw2, g->db1, g->db2, nullptr, cs);
  attn_bwd_impl(z, causal, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                nullptr, nullptr, g->dwqkv, g->dbqkv, g->dwout, g->dbout, nullptr, cs);
  for (tp_bf16* q : {g->dln1_g, g->dln1_b, g->dln2_g, g->dln2_b})
    if (q) cudaMemsetAsync(q, 0, (size_t)z.D * 2, cs);
  return cuda_status(cudaGetLastError());
}

}  // namespace
}  // namespace tp

extern "C" {

tp_status tp_layer_fwd(const tp_dims* dims, const tp_bf16* x, const tp_layer_params* p,
                       const tp_layer_acts* a, tp_bf16* y, void* ws, size_t ws_bytes, tp_stream s) {
  tp_status st = check_layer(dims);
  if (st != TP_OK) return st;
  if (has_tokens(dims) && !all_set(x, y)) return TP_ERR_INVALID_ARG;
  if ((st = check_layer_ptrs(p, a, has_tokens(dims))) != TP_OK) return st;
  if (!all_aligned(x, y)) return TP_ERR_MISALIGNED;
  const Sizes z = sizes_of(*dims);
  cudaStream_t cs = (cudaStream_t)s;
  if (z.T == 0) return TP_OK;
  if ((st = check_ws(ws, ws_bytes, layer_fwd_ws(z))) != TP_OK) return st;
  uint16_t* w16 = a->wqkv16 != nullptr ? a->wqkv16 : static_cast<uint16_t*>(ws);
  if ((st = launch_cast_f16(p->wqkv, (size_t)(z.D * 3 * z.D), w16, cs)) != TP_OK) return st;
  return layer_fwd_core(z, dims, x, p, a, y, w16, cs);
}

tp_status tp_layer_bwd(const tp_dims* dims, const tp_bf16* x, const tp_layer_params* p,
                       const tp_layer_acts* a, const tp_bf16* dy, tp_bf16* dx,
                       const tp_layer_grads* g, void* ws, size_t ws_bytes, tp_stream s) {
  DstLimitPin pin;   // one dS^T limit for the whole call
  tp_status st = check_layer(dims);
  if (st != TP_OK) return st;
  if ((st = check_layer_ptrs(p, a, has_tokens(dims))) != TP_OK) return st;
  if ((st = check_layer_grads(dims, x, dy, dx, g)) != TP_OK) return st;
  const Sizes z = sizes_of(*dims);
  const size_t need = z.T ? layer_bwd_ws(z) : 0;
  if ((st = check_ws(ws, ws_bytes, need)) != TP_OK) return st;
  cudaStream_t cs = (cudaStream_t)s;
  if (z.T == 0) return layer_bwd_empty(z, dims->causal, g, cs);
  return layer_bwd_core(z, dims, x, p, a, dy, dx, g, ws, cs);
}

tp_status tp_layer_bwd_notify(const tp_dims* dims, const tp_bf16* x, const tp_layer_params* p,
                              const tp_layer_acts* a, const tp_bf16* dy, tp_bf16* dx,
                              const tp_layer_grads* g, const tp_grad_ready* ready, void* ws,
                              size_t ws_bytes, tp_stream s) {
  DstLimitPin pin;   // one dS^T limit for the whole call
  tp_status st = check_layer(dims);
  if (st != TP_OK) return st;
  if ((st = check_layer_ptrs(p, a, has_tokens(dims))) != TP_OK) return st;
  if ((st = check_layer_grads(dims, x, dy, dx, g)) != TP_OK) return st;
  const Sizes z = sizes_of(*dims);
  const size_t need = z.T ? layer_bwd_ws(z) : 0;
  if ((st = check_ws(ws, ws_bytes, need)) != TP_OK) return st;
  cudaStream_t cs = (cudaStream_t)s;
  if (z.T == 0) {
    if ((st = layer_bwd_empty(z, dims->causal, g, cs)) != TP_OK) return st;
    if (ready) {
      for (void* ev : {ready->mlp, ready->attn, ready->ln1})
        if ((st = record_ready(ev, cs)) != TP_OK) return st;
    }
    return TP_OK;
  }
  return layer_bwd_core(z, dims, x, p, a, dy, dx, g, ws, cs, ready);
}

tp_status tp_layer_fwd_nosave(const tp_dims* dims, const tp_bf16* x, const tp_layer_params* p,
                              tp_bf16* y, void* ws, size_t ws_bytes, tp_stream s) {
  tp_status st = check_layer(dims);
  if (st != TP_OK) return st;
  if ((long long)dims->batch * dims->seq > 0 && !all_set(x, y)) return TP_ERR_INVALID_ARG;
  if ((st = check_layer_params(p)) != TP_OK) return st;
  if (!all_aligned(x, y)) return TP_ERR_MISALIGNED;
  const Sizes z = sizes_of(*dims);
  cudaStream_t cs = (cudaStream_t)s;
  if (z.T == 0) return TP_OK;
  if ((st = check_ws(ws, ws_bytes, layer_fwd_nosave_ws(z))) != TP_OK) return st;
  Carver c(ws);
  uint16_t* w16 = c.take<uint16_t>((size_t)(z.D * 3 * z.D));
  c.off = align_up(layer_fwd_ws(z), 256);
  const tp_layer_acts a = carve_layer_acts(c, z);
  if ((st = launch_cast_f16(p->wqkv, (size_t)(z.D * 3 * z.D), w16, cs)) != TP_OK) return st;
  return layer_fwd_core(z, dims, x, p, &a, y, w16, cs);
}

tp_status tp_layer_bwd_recompute(const tp_dims* dims, const tp_bf16* x, const tp_layer_params* p,
                                 const tp_bf16* dy, tp_bf16* dx, const tp_layer_grads* g,
                                 void* ws, size_t ws_bytes, tp_stream s) {
  DstLimitPin pin;   // one dS^T limit for the whole call
  tp_status st = check_layer(dims);
  if (st != TP_OK) return st;
  if ((st = check_layer_params(p)) != TP_OK) return st;
  if ((st = check_layer_grads(dims, x, dy, dx, g)) != TP_OK) return st;
  const Sizes z = sizes_of(*dims);
  const size_t need = z.T ? layer_bwd_recompute_ws(z) : 0;
  if ((st = check_ws(ws, ws_bytes, need)) != TP_OK) return st;
  cudaStream_t cs = (cudaStream_t)s;
  if (z.T == 0) return layer_bwd_empty(z, dims->causal, g, cs);
  Carver c(ws);
  const tp_layer_acts a = carve_layer_acts(c, z);
  c.off = align_up(layer_acts_ws(z), 256);
  void* bws = c.take<uint8_t>(layer_bwd_ws(z));
  uint16_t* w16 = static_cast<uint16_t*>(bws);
  if ((st = launch_cast_f16(p->wqkv, (size_t)(z.D * 3 * z.D), w16, cs)) != TP_OK) return st;
  if ((st = layer_fwd_core(z, dims, x, p, &a, nullptr, w16, cs)) != TP_OK) return st;
  tp_layer_acts ar = a;
  ar.wqkv16 = w16;   // the recomputed forward's copy serves the backward
  return layer_bwd_core(z, dims, x, p, &ar, dy, dx, g, bws, cs);
}

// ------------------------------------------------------------------ post-LN layer
static tp_status check_postln_ptrs(const tp_layer_params* p, const tp_postln_acts* a, bool tok) {
  if (!p || !a) return TP_ERR_INVALID_ARG;
  if (!all_set(p->ln1_g, p->ln1_b, p->wqkv, p->wout, p->ln2_g, p->ln2_b, p->w1, p->w2))
    return TP_ERR_INVALID_ARG;
  if (tok && !all_set(a->z1, a->mean1, a->rstd1, a->qkv, a->o, a->lse, a->h, a->z2, a->mean2,
                      a->rstd2, a->a, a->hact))
    return TP_ERR_INVALID_ARG;
  if (!all_aligned(p->ln1_g, p->ln1_b, p->wqkv, p->bqkv, p->wout, p->bout, p->ln2_g, p->ln2_b,
                   p->w1, p->b1, p->w2, p->b2))
    return TP_ERR_MISALIGNED;
  if (!all_aligned(a->z1, a->qkv, a->o, a->lse, a->h, a->z2, a->a, a->hact)) return TP_ERR_MISALIGNED;
  return TP_OK;
}

tp_status tp_postln_layer_fwd(const tp_dims* dims, const tp_bf16* x, const tp_layer_params* p,
                              const tp_postln_acts* a, tp_bf16* y, void* ws, size_t ws_bytes,
                              tp_stream s) {
  tp_status st = check_layer(dims);
  if (st != TP_OK) return st;
  if (has_tokens(dims) && !all_set(x, y)) return TP_ERR_INVALID_ARG;
  if ((st = check_postln_ptrs(p, a, has_tokens(dims))) != TP_OK) return st;
  if (!all_aligned(x, y)) return TP_ERR_MISALIGNED;
  const Sizes z = sizes_of(*dims);
  cudaStream_t cs = (cudaStream_t)s;
  if (z.T == 0) return TP_OK;
  if ((st = check_ws(ws, ws_bytes, postln_fwd_ws(z))) != TP_OK) return st;
  Carver c(ws);
  uint16_t* x16 = c.take<uint16_t>((size_t)(z.T * z.D));
  uint16_t* w16 = c.take<uint16_t>((size_t)(z.D * 3 * z.D));
  if ((st = launch_cast_f16(x, (size_t)(z.T * z.D), x16, cs)) != TP_OK) return st;
  if ((st = launch_cast_f16(p->wqkv, (size_t)(z.D * 3 * z.D), w16, cs)) != TP_OK) return st;
  // z1 = x + Attn(x); h = LN1(z1); z2 = h + MLP(h); y = LN2(z2)
  if ((st = attn_fwd_impl(z, dims->causal, x16, w16, p->bqkv, p->wout, p->bout, x, a->z1, a->qkv,
                          a->o, a->lse, cs)) != TP_OK)
    return st;
  if ((st = launch_layernorm_fwd(a->z1, p->ln1_g, p->ln1_b, z.T, (int)z.D, dims->ln_eps, a->h,
                                 a->mean1, a->rstd1, cs)) != TP_OK)
    return st;
  if ((st = mlp_fwd_impl(z, a->h, p->w1, p->b1, p->w2, p->b2, a->h, a->z2, a->a, a->hact, cs)) !=
      TP_OK)
    return st;
  return launch_layernorm_fwd(a->z2, p->ln2_g, p->ln2_b, z.T, (int)z.D, dims->ln_eps, y, a->mean2,
                              a->rstd2, cs);
}

tp_status tp_postln_layer_bwd(const tp_dims* dims, const tp_bf16* x, const tp_layer_params* p,
                              const tp_postln_acts* a, const tp_bf16* dy, tp_bf16* dx,
                              const tp_layer_grads* g, void* ws, size_t ws_bytes, tp_stream s) {
  DstLimitPin pin;   // one dS^T limit for the whole call
  tp_status st = check_layer(dims);
  if (st != TP_OK) return st;
  if ((st = check_postln_ptrs(p, a, has_tokens(dims))) != TP_OK) return st;
  if ((st = check_layer_grads(dims, x, dy, dx, g)) != TP_OK) return st;
  const Sizes z = sizes_of(*dims);
  cudaStream_t cs = (cudaStream_t)s;
  if (z.T == 0) {
    mlp_bwd_impl(z, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, g->dw1,
                 g->dw2, g->db1, g->db2, nullptr, cs);
    attn_bwd_impl(z, dims->causal, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                  nullptr, nullptr, g->dwqkv, g->dbqkv, g->dwout, g->dbout, nullptr, cs);
    for (tp_bf16* q : {g->dln1_g, g->dln1_b, g->dln2_g, g->dln2_b})
      if (q) cudaMemsetAsync(q, 0, (size_t)z.D * 2, cs);
    return cuda_status(cudaGetLastError());
  }
  if ((st = check_ws(ws, ws_bytes, postln_bwd_ws(z))) != TP_OK) return st;
  Carver c(ws);
  uint16_t* x16 = c.take<uint16_t>((size_t)(z.T * z.D));
  uint16_t* w16 = c.take<uint16_t>((size_t)(z.D * 3 * z.D));
  c.off = align_up(attn_fwd_ws(z), 256);
  uint16_t* d16 = c.take<uint16_t>((size_t)(z.T * z.D));   // dz2, then dz1 (GEMM operand)
  float* d32 = c.take<float>((size_t)(z.T * z.D));          // dz2, then dz1 (residual carry)
  float* dh32 = c.take<float>((size_t)(z.T * z.D));
  float* lnp = c.take<float>(layernorm_bwd_partial_floats(z.T, (int)z.D));
  const size_t sub = mlp_bwd_ws(z) > attn_bwd_core_ws(z) ? mlp_bwd_ws(z) : attn_bwd_core_ws(z);
  void* subws = c.take<uint8_t>(sub);
  // y = LN2(z2): dz2 = LN2^T(dy).  z2 = h + MLP(h): dh = dz2 + MLP^T(dz2).
  if ((st = launch_layernorm_bwd(dy, a->z2, p->ln2_g, a->mean2, a->rstd2, nullptr, z.T, (int)z.D,
                                 d16, g->dln2_g, g->dln2_b, lnp, cs, d32)) != TP_OK)
    return st;
  if ((st = mlp_bwd_impl(z, a->h, p->w1, p->w2, a->a, a->hact, d16, nullptr, nullptr, g->dw1,
                         g->dw2, g->db1, g->db2, subws, cs, d32, dh32)) != TP_OK)
    return st;
  // h = LN1(z1): dz1 = LN1^T(dh).  z1 = x + Attn(x): dx = dz1 + Attn^T(dz1).
  if ((st = launch_layernorm_bwd_f32(dh32, a->z1, p->ln1_g, a->mean1, a->rstd1, z.T, (int)z.D,
                                     d16, d32, g->dln1_g, g->dln1_b, lnp, cs)) != TP_OK)
    return st;
  if ((st = launch_cast_f16(x, (size_t)(z.T * z.D), x16, cs)) != TP_OK) return st;
  if ((st = launch_cast_f16(p->wqkv, (size_t)(z.D * 3 * z.D), w16, cs)) != TP_OK) return st;
  return attn_bwd_impl(z, dims->causal, x16, w16, p->wout, a->qkv, a->o, a->lse, d16, nullptr, dx,
                       g->dwqkv, g->dbqkv, g->dwout, g->dbout, subws, cs, d32);
}

}  // extern "C"
