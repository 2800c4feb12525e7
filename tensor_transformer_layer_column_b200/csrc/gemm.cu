// Host side of the tcgen05 GEMM: tensor-map encoding and launch.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "gemm_sm100.cuh"
#include "internal.h"

namespace tp {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D 16-bit tensor map with 128-byte swizzle; out-of-range elements read as 0.
bool encode_operand(CUtensorMap* map, const OperandDesc& d, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d.inner, (cuuint64_t)d.outer, (cuuint64_t)d.shards};
  const long long shard_stride = d.shards > 1 ? d.shard_stride : d.ld * d.outer;
  const cuuint64_t strides[2] = {(cuuint64_t)d.ld * 2, (cuuint64_t)shard_stride * 2};
  const cuuint32_t box[3] = {64, box_outer, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, d.f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(d.ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// MN-major operand staged chunk-interleaved: a 5-D view (64 of MN, 8 K rows,
// MN/64 chunks, K/8 groups, shards) whose box {64, 8, chunks, 8, 1} lands in
// shared memory as [K group][chunk][8 rows x 128 B].  Needs MN % 64 == 0 and
// K % 8 == 0 so that the view covers exactly the tensor.
bool interleave_ok(const OperandDesc& d) {
  return d.mn_major && d.inner % 64 == 0 && d.outer % 8 == 0;
}

bool encode_operand_il(CUtensorMap* map, const OperandDesc& d, uint32_t chunks) {
  auto fn = encode_fn();
  if (!fn) return false;
  const long long shard_stride = d.shards > 1 ? d.shard_stride : d.ld * d.outer;
  const cuuint64_t dims[5] = {64, 8, (cuuint64_t)(d.inner / 64), (cuuint64_t)(d.outer / 8),
                              (cuuint64_t)d.shards};
  const cuuint64_t strides[4] = {(cuuint64_t)d.ld * 2, 128, (cuuint64_t)d.ld * 16,
                                 (cuuint64_t)shard_stride * 2};
  const cuuint32_t box[5] = {64, 8, chunks, 8, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, d.f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
                  const_cast<void*>(d.ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool A_MN, bool B_MN>
tp_status launch_inst(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& args,
                      int grid, double flops, cudaStream_t stream) {
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  auto kern = gemm_bf16_sm100<A_MN, B_MN>;
  if (dev < 64 && !configured[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GEMM_SMEM_BYTES) != cudaSuccess)
      return TP_ERR_CUDA;
    configured[dev] = true;
  }
  {
    TraceScope ts(stream, TK_GEMM, flops);
    kern<<<grid, GEMM_THREADS, GEMM_SMEM_BYTES, stream>>>(ta, tb, args);
  }
  return cuda_status(cudaGetLastError());
}

// CTA-pair kernel: clusters of 2 CTAs, one 256 x 256 tile per cluster at a
// time, over the tiles of `args` and then of `args2` (num_tiles 0: none).
template <bool A_MN, bool B_MN>
tp_status launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& args,
                      const CUtensorMap& ta2, const CUtensorMap& tb2, const GemmArgs& args2,
                      double flops, cudaStream_t stream) {
  static int max_clusters[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  auto kern = gemm_pair_sm100<A_MN, B_MN>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see launch_pdl
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = GP_SMEM_BYTES;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (dev < 0 || dev >= 64) return TP_ERR_CUDA;
  if (max_clusters[dev] == 0) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GP_SMEM_BYTES) !=
        cudaSuccess)
      return TP_ERR_CUDA;
    int n = 0;
    cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) return TP_ERR_CUDA;
    max_clusters[dev] = n;
  }
  const int tiles = args.num_tiles + args2.num_tiles;
  const int clusters = tiles < max_clusters[dev] ? tiles : max_clusters[dev];
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.numAttrs = 2;
  {
    TraceScope ts(stream, TK_GEMM, flops);
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, args, ta2, tb2, args2) != cudaSuccess)
      return TP_ERR_CUDA;
  }
  return cuda_status(cudaGetLastError());
}

// Tensor maps and kernel arguments of one product; *pair: the CTA-pair
// kernel runs it (one 128-row block does not cover M).
tp_status prepare(const GemmProblem& g, CUtensorMap* ta, CUtensorMap* tb, GemmArgs* out,
                  bool* pair_out, double* flops, bool force_pair = false) {
  if (g.a.f16 != g.b.f16) return TP_ERR_INVALID_ARG;       // one MMA takes one operand type
  // fp32 residual / output: plain linear epilogue, no fp16 store.
  if ((g.out_f32 || g.aux_f32) && (g.epi != EPI_LINEAR || g.out_f16)) return TP_ERR_INVALID_ARG;
  if (g.colpart != nullptr && g.m_shards != 1) return TP_ERR_INVALID_ARG;
  // Pairs of CTAs (256-row tiles) unless one 128-row block covers M (or the
  // caller asks for the pair kernel: rows past Mt read as zero and are not stored).
  const bool pair = force_pair || g.Mt > GEMM_BM;
  const bool a_il = interleave_ok(g.a), b_il = interleave_ok(g.b);
  if (a_il ? !encode_operand_il(ta, g.a, GEMM_BM / 64)
           : !encode_operand(ta, g.a, g.a.mn_major ? 64 : GEMM_BM))
    return TP_ERR_CUDA;
  const uint32_t b_rows = pair ? 128 : GEMM_BN;
  if (b_il ? !encode_operand_il(tb, g.b, b_rows / 64)
           : !encode_operand(tb, g.b, g.b.mn_major ? 64 : b_rows))
    return TP_ERR_CUDA;

  GemmArgs a{};
  a.m_shards = g.m_shards;
  a.n_shards = g.n_shards;
  a.Mt = g.Mt;
  a.Nt = g.Nt;
  const int bm = pair ? GP_BM : GEMM_BM, bn = pair ? GP_BN : GEMM_BN;
  a.mb_per_shard = (g.Mt + bm - 1) / bm;
  a.nb_per_shard = (g.Nt + bn - 1) / bn;
  a.k_shards = g.k_shards;
  a.kb_per_shard = (g.Kt + GEMM_BK - 1) / GEMM_BK;
  a.a_src = g.a.src;
  a.b_src = g.b.src;
  const long long tiles = (long long)a.m_shards * a.mb_per_shard * a.n_shards * a.nb_per_shard;
  a.num_tiles = (int)tiles;
  a.group_m = 8;
  a.epi = g.epi;
  a.c = static_cast<__nv_bfloat16*>(g.c);
  a.c2 = static_cast<__nv_bfloat16*>(g.c2);
  a.aux = static_cast<const __nv_bfloat16*>(g.aux);
  a.bias = static_cast<const __nv_bfloat16*>(g.bias);
  a.c_ms = g.c_ms;
  a.c_ns = g.c_ns;
  a.ldc = g.ldc;
  a.err = error_word();
  a.idesc = idesc_f32acc(pair ? GP_BM : GEMM_BM, pair ? GP_BN : GEMM_BN, g.a.mn_major,
                         g.b.mn_major, g.a.f16);
  a.out_f16 = g.out_f16 ? 1 : 0;
  a.out_f32 = g.out_f32 ? 1 : 0;
  a.aux_f32 = g.aux_f32 ? 1 : 0;
  a.a_il = a_il ? 1 : 0;
  a.b_il = b_il ? 1 : 0;
  a.colpart = g.colpart;
  a.colpart_ld = (long long)g.n_shards * g.Nt;
  *out = a;
  *pair_out = pair;
  *flops = 2.0 * g.m_shards * (double)g.Mt * g.n_shards * (double)g.Nt * g.k_shards * (double)g.Kt;
  return TP_OK;
}

tp_status pair_dispatch(bool a_mn, bool b_mn, const CUtensorMap& ta, const CUtensorMap& tb,
                        const GemmArgs& a, const CUtensorMap& ta2, const CUtensorMap& tb2,
                        const GemmArgs& a2, double flops, cudaStream_t stream) {
  if (!a_mn && b_mn) return launch_pair<false, true>(ta, tb, a, ta2, tb2, a2, flops, stream);
  if (!a_mn && !b_mn) return launch_pair<false, false>(ta, tb, a, ta2, tb2, a2, flops, stream);
  if (a_mn && b_mn) return launch_pair<true, true>(ta, tb, a, ta2, tb2, a2, flops, stream);
  return launch_pair<true, false>(ta, tb, a, ta2, tb2, a2, flops, stream);
}

}  // namespace

tp_status launch_gemm(const GemmProblem& g, cudaStream_t stream) {
  if (g.Mt <= 0 || g.Nt <= 0 || g.Kt <= 0) return TP_OK;   // empty product: nothing to do
  CUtensorMap ta, tb;
  GemmArgs a;
  bool pair = false;
  double flops = 0;
  tp_status s = prepare(g, &ta, &tb, &a, &pair, &flops);
  if (s != TP_OK) return s;
  if (pair) {
    GemmArgs none = a;
    none.num_tiles = 0;
    return pair_dispatch(g.a.mn_major, g.b.mn_major, ta, tb, a, ta, tb, none, flops, stream);
  }
  const long long tiles = a.num_tiles;
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  if (!g.a.mn_major && g.b.mn_major) return launch_inst<false, true>(ta, tb, a, grid, flops, stream);
  if (!g.a.mn_major && !g.b.mn_major) return launch_inst<false, false>(ta, tb, a, grid, flops, stream);
  if (g.a.mn_major && g.b.mn_major) return launch_inst<true, true>(ta, tb, a, grid, flops, stream);
  return launch_inst<true, false>(ta, tb, a, grid, flops, stream);
}

tp_status launch_gemm2(const GemmProblem& g1, const GemmProblem& g2, cudaStream_t stream) {
  const bool e1 = g1.Mt <= 0 || g1.Nt <= 0 || g1.Kt <= 0;
  const bool e2 = g2.Mt <= 0 || g2.Nt <= 0 || g2.Kt <= 0;
  // One launch of the pair kernel when the operand majors agree (each tile's
  // products take its own problem's operand type; a product with M <= 128
  // runs on 256-row tiles here), so that the launch sequence does not depend
  // on the sizes; otherwise one after the other.
  if (e1 || e2 || g1.a.mn_major != g2.a.mn_major || g1.b.mn_major != g2.b.mn_major) {
    tp_status s = launch_gemm(g1, stream);
    return s != TP_OK ? s : launch_gemm(g2, stream);
  }
  CUtensorMap ta1, tb1, ta2, tb2;
  GemmArgs a1, a2;
  bool p1 = false, p2 = false;
  double f1 = 0, f2 = 0;
  tp_status s = prepare(g1, &ta1, &tb1, &a1, &p1, &f1, true);
  if (s != TP_OK) return s;
  if ((s = prepare(g2, &ta2, &tb2, &a2, &p2, &f2, true)) != TP_OK) return s;
  return pair_dispatch(g1.a.mn_major, g1.b.mn_major, ta1, tb1, a1, ta2, tb2, a2, f1 + f2, stream);
}

}  // namespace tp
