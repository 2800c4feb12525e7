// Declarations shared by the translation units of libtplayer.so (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>
#include <utility>

#include "pdl.cuh"
#include "tp_layer.h"

namespace tp {

// One GEMM operand as a 3-D tensor (inner, outer, shards), row-major, bf16.
//   K-major operand : inner = K extent, outer = M (or N) extent;
//   MN-major operand: inner = M (or N) extent, outer = K extent.
// src selects what indexes the shard dimension: nothing, the K walk, or the
// operand's own M/N shard.
struct OperandDesc {
  const void* ptr;
  bool mn_major;
  bool f16;                  // element type: fp16 (true) or bf16 (false)
  int src;                   // ShardSrc
  long long inner, outer, shards;
  long long ld;              // elements between consecutive outer indices
  long long shard_stride;    // elements between consecutive shards
};

struct GemmProblem {
  int m_shards, n_shards, Mt, Nt;
  int k_shards, Kt;
  OperandDesc a, b;
  int epi;                   // EpiKind
  void* c;
  void* c2;
  const void* aux;
  const void* bias;
  long long c_ms, c_ns, ldc;
  bool out_f16;              // store C / C2 as fp16
  bool out_f32;              // store C as fp32 (EPI_LINEAR only)
  bool aux_f32;              // aux is an fp32 residual (EPI_LINEAR only)
  // When set (one M shard only): per 32-row group column sums of C, fp32
  // [ceil(Mt / 32)][n_shards * Nt]; reduce them with launch_colsum_reduce.
  float* colpart = nullptr;
};

tp_status launch_gemm(const GemmProblem& g, cudaStream_t stream);
// g1 then g2 in one launch of the CTA-pair kernel when both run on it with
// the same operand majors (the tiles of both fill the clusters' rounds
// together; each keeps its own operand type); otherwise two launches.  The
// products must not depend on each other.
tp_status launch_gemm2(const GemmProblem& g1, const GemmProblem& g2, cudaStream_t stream);

// Launch with the programmatic-serialization attribute (see pdl.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Host validation of tp_dims shared by the entry points (status before any launch).
tp_status check_common(const tp_dims* d);
tp_status check_mlp(const tp_dims* d);
tp_status check_attn(const tp_dims* d);
tp_status check_layer(const tp_dims* d);

// Device error word of the current device (bounded-wait timeouts).
unsigned int* error_word();
int sm_count();

// Column sums of S stacked [rows][cols] bf16 matrices into bf16 out[S][cols]
// (fp32 accumulation, deterministic two-pass over `partial`, an fp32 scratch
// of colsum_partial_floats(S, rows, cols) floats).
size_t colsum_partial_floats(long long S, long long rows, long long cols);
tp_status launch_colsum_stacked(const uint16_t* x, long long S, long long rows, long long cols,
                                uint16_t* out, float* partial, cudaStream_t stream,
                                bool in_f16 = false);
// out[c] = bf16( sum over r of partial[r][c] ), r = 0..rows-1 in order.
tp_status launch_colsum_reduce(const float* partial, long long rows, long long cols, uint16_t* out,
                               cudaStream_t stream);

tp_status launch_layernorm_fwd(const uint16_t* x, const uint16_t* g, const uint16_t* b,
                               long long rows, int D, float eps, uint16_t* y, float* mean,
                               float* rstd, cudaStream_t stream, bool out_f16 = false);
// Row blocks of the LayerNorm backward (2 per SM, at most one per row); the
// dgamma/dbeta partials hold 2 * D floats per block.
int layernorm_bwd_blocks(long long rows);
// Partial floats of the LayerNorm backward: nk rows of D per block (2: dgamma,
// dbeta; 3: also the column sums of dres, see launch_layernorm_bwd).
size_t layernorm_bwd_partial_floats(long long rows, int D, int nk = 2);
// dres_sum (needs dres; partial sized with nk = 3): the column sums of dres,
// bf16 [D] -- the bias gradient of the product whose output gradient dres is.
tp_status launch_layernorm_bwd(const uint16_t* dy, const uint16_t* x, const uint16_t* g,
                               const float* mean, const float* rstd, const uint16_t* dres,
                               long long rows, int D, uint16_t* dx, uint16_t* dg, uint16_t* db,
                               float* partial, cudaStream_t stream, float* dx32 = nullptr,
                               uint16_t* dres_sum = nullptr);

// fp32 upstream gradient dy; dx is written bf16 and, when dx32 is set, also fp32.
tp_status launch_layernorm_bwd_f32(const float* dy, const uint16_t* x, const uint16_t* g,
                                   const float* mean, const float* rstd, long long rows, int D,
                                   uint16_t* dx, float* dx32, uint16_t* dg, uint16_t* db,
                                   float* partial, cudaStream_t stream);

tp_status launch_layernorm_bwd_blocks(const uint16_t* dy, const uint16_t* x, const uint16_t* g,
                                      const float* mean, const float* rstd, const uint16_t* dres,
                                      long long rows, int D, uint16_t* dx, uint16_t* dg,
                                      uint16_t* db, int nb, float* partial, cudaStream_t stream);

// Per-head causal attention over the shard-packed qkv [t][T][3Dt].
tp_status launch_attn_fwd(const uint16_t* qkv, uint16_t* o, float* lse, int B, int S, int H,
                          int dh, int t, int causal, cudaStream_t stream);
size_t attn_bwd_scratch_bytes(int B, int S, int H, int dh);
// Largest dS^T array (bytes) the attention backward keeps for its dQ kernel;
// returns the previous limit.
size_t attn_set_dst_limit(size_t max_bytes);
// While one is in scope, the calling thread reads the limit as it was when
// the outermost one was made: a library call that sizes, checks and carves a
// workspace and then launches into it sees one value, whatever another
// thread sets meanwhile.
struct DstLimitPin {
  DstLimitPin();
  ~DstLimitPin();
  DstLimitPin(const DstLimitPin&) = delete;
  DstLimitPin& operator=(const DstLimitPin&) = delete;
  bool outer_;
};
// colpart (may be null): column sums of dqkv, fp32 [B * ceil(S / 32)][t * 3Dt] (one
// partial row per 32 rows of a batch element), for launch_colsum_reduce.
tp_status launch_attn_bwd(const uint16_t* qkv, const uint16_t* o, const float* lse,
                          const uint16_t* dout, uint16_t* dqkv, int B, int S, int H, int dh, int t,
                          int causal, void* scratch, cudaStream_t stream,
                          float* colpart = nullptr);
inline long long attn_colpart_rows(long long B, long long S) { return B * ((S + 31) / 32); }

tp_status launch_shard_cols(const uint16_t* src, int rows, int cols, int t, uint16_t* dst,
                            bool inverse, cudaStream_t stream);
tp_status launch_shard_qkv(const uint16_t* src, int rows, int hidden, int t, uint16_t* dst,
                           bool inverse, cudaStream_t stream);
tp_status launch_copy(const uint16_t* src, size_t n, uint16_t* dst, cudaStream_t stream);
// bf16 -> fp16 element copy (n elements); values beyond the fp16 range set
// the device error word to 0x301.
tp_status launch_cast_f16(const uint16_t* src, size_t n, uint16_t* dst, cudaStream_t stream);

// Kernel classes reported by the launch trace (tp_trace_begin).
enum TraceKind : int {
  TK_GEMM = 0, TK_ATTN_FWD = 1, TK_ATTN_BWD_PREP = 2, TK_ATTN_BWD_DKDV = 3, TK_ATTN_BWD_DQ = 4,
  TK_LN_FWD = 5, TK_LN_BWD = 6, TK_LN_PARAM = 7, TK_COLSUM = 8, TK_LAYOUT = 9, TK_CAST = 10,
  TK_FINISH = 11,
};

// Brackets one kernel launch with the trace's events when a trace is open.
class TraceScope {
 public:
  TraceScope(cudaStream_t stream, int kind, double flops = 0.0);
  ~TraceScope();
  TraceScope(const TraceScope&) = delete;
  TraceScope& operator=(const TraceScope&) = delete;

 private:
  cudaStream_t stream_;
  int slot_;
};

inline tp_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TP_OK : TP_ERR_CUDA; }

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---------------------------------------------------------------- host-side argument checks
inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Every non-null pointer 16-byte aligned.
template <typename... P>
bool all_aligned(P... ps) {
  bool ok = true;
  ((ok = ok && (ps == nullptr || al16(ps))), ...);
  return ok;
}

template <typename... P>
bool all_set(P... ps) {
  bool ok = true;
  ((ok = ok && ps != nullptr), ...);
  return ok;
}

inline bool supported_t(int t) { return t == 1 || t == 2 || t == 4 || t == 8; }

// Workspace carving: consecutive 256-byte aligned slices.
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* p) : base(static_cast<uint8_t*>(p)) {}
  template <typename T>
  T* take(size_t count) {
    off = align_up(off, 256);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

inline tp_status check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return TP_OK;
  if (ws == nullptr || have < need) return TP_ERR_WORKSPACE;
  if (!al16(ws)) return TP_ERR_MISALIGNED;
  return TP_OK;
}

}  // namespace tp
