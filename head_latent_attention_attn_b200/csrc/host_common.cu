// host_common.cu - tensor-map encoding through the driver entry point and dims checks.
#include <cudaTypedefs.h>

#include <mutex>

#include "host_common.h"

namespace mla {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

void load_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess) {
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
}
}  // namespace

bool encode_bf16_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box,
                     CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode) return false;
  cuuint64_t gdim[5];
  cuuint64_t gstride[4];
  cuuint32_t bdim[5];
  cuuint32_t estride[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estride[i] = 1;
    if (i + 1 < rank) gstride[i] = strides_bytes[i];
  }
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base),
                        gdim, gstride, bdim, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

mla_status check_dims(const mla_dims* d) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->num_heads <= 0 || d->num_kv_groups <= 0 || d->num_heads % d->num_kv_groups != 0)
    return MLA_ERR_INVALID_ARG;
  if (d->kv_lora_rank <= 0 || d->kv_lora_rank % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (d->qk_nope_dim <= 0 || d->qk_nope_dim % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (d->v_head_dim <= 0 || d->v_head_dim % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (d->rope_dim < 0 || d->rope_dim % 2 != 0) return MLA_ERR_INVALID_ARG;
  if (row_width(d) % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (d->page_size <= 0) return MLA_ERR_INVALID_ARG;
  if (!(d->softmax_scale > 0.0f) || d->softmax_scale != d->softmax_scale) return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

}  // namespace mla
