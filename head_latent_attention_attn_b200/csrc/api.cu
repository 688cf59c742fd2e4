// api.cu - the extern "C" boundary of libmla.so (declared in include/mla.h): argument
// validation, tensor-map encoding and launch planning. No allocation happens here; every
// buffer is the caller's.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "host_common.h"
#include "kernels.h"
#include "ptx.cuh"

using namespace mla;

namespace {

// Self-test of the device error path: one warp waits, with the bounded wait of every kernel
// here, on an mbarrier that nothing arrives on; the wait gives up, sets the CTA's abort flag
// and ORs MLA_DEVERR_TIMEOUT into the error word, and the kernel returns.
__global__ void __launch_bounds__(32) mla_selftest_wait_kernel(int32_t* dev_error) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtx wc{&abort_flag, dev_error};
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, wc);   // phase 0 never completes
  __syncthreads();
}

constexpr int kMaxSmem = 232448;  // 227 KB opt-in dynamic shared memory per CTA



inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

// Clusters of two pair-kernel CTAs that fit on the current device at once, cached per
// (device, shared-memory size); falls back to half the SM count if the query fails.
int pair_clusters(size_t smem) {
  static std::mutex mu;
  static int cache_dev[16], cache_val[16];
  static size_t cache_smem[16];
  static int cache_n = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return num_sms() / 2;
  }
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < cache_n; ++i)
    if (cache_dev[i] == dev && cache_smem[i] == smem) return cache_val[i];
  int n = decode_pair_max_clusters(smem);
  if (n <= 0) n = num_sms() / 2;
  n = std::min(n, num_sms() / 2);
  if (cache_n < 16) {
    cache_dev[cache_n] = dev;
    cache_smem[cache_n] = smem;
    cache_val[cache_n] = n;
    ++cache_n;
  }
  return n;
}

int pow2_at_least(int x, int lo) {
  int v = lo;
  while (v < x) v <<= 1;
  return v;
}

// Launch geometry of one mla_decode_attn problem.
struct DecodePlan {
  int ncol, col_groups, units, nblk, nch, slot_blocks, nslot, npt, tmem_cols, grid;
  int pair;        // 1: blocks of 128 rows on clusters of two CTAs that split the latent
  int rope_half;   // rotary columns per CTA of a pair
  int vgrid;       // work ranges (CTAs, or clusters for the pair kernel)
  size_t smem;
  size_t ws_bytes;
  size_t range_off, unit_start_off, part_lse_off, part_o_off;
};


size_t align256(size_t x) { return (x + 255) / 256 * 256; }

mla_status plan_decode(const mla_dims* d, int32_t batch, int32_t q_len, int32_t max_seq_len,
                       int32_t num_splits, DecodePlan* P) {
  mla_status st = check_dims(d);
  if (st != MLA_OK) return st;
  if (batch < 0 || q_len <= 0 || max_seq_len < q_len || num_splits < 0)
    return MLA_ERR_INVALID_ARG;
  if (d->page_size != kDecodeTok) return MLA_ERR_UNSUPPORTED;
  const int r = d->kv_lora_rank;
  const int D = row_width(d);
  if (r > 512 || D > 64 * kDecodeMaxBlk) return MLA_ERR_UNSUPPORTED;
  const int64_t qH = int64_t(q_len) * d->num_heads;
  const int R = d->num_kv_groups * d->rope_dim;
  // More than 64 rows per sequence: 128-row blocks on clusters of two CTAs that split the
  // latent (r a multiple of 128, rotary half of 16, 32 or 64 columns); else blocks of
  // 16, 32 or 64 rows, one CTA each.
  P->pair = (qH > 64 && r % 128 == 0 && (R == 32 || R == 64 || R == 128)) ? 1 : 0;
  P->rope_half = R / 2;
  P->ncol = P->pair ? kPairRows : (qH <= 16 ? 16 : (qH <= 32 ? 32 : 64));
  P->col_groups = int((qH + P->ncol - 1) / P->ncol);
  const int64_t units = int64_t(std::max(batch, 1)) * P->col_groups;
  if (units > (int64_t(1) << 24)) return MLA_ERR_UNSUPPORTED;
  P->units = int(units);
  P->nblk = (D + 63) / 64;
  P->nch = (r + 127) / 128;
  P->slot_blocks = std::max(P->nblk, 2 * P->nch);
  P->nslot = 0;
  P->npt = 1;
  if (P->pair) {
    P->tmem_cols = 512;
    for (int ns = kPairMaxSlots; ns >= 2 && P->nslot == 0; --ns)
      if (decode_pair_smem_bytes(r, P->rope_half, ns) <= size_t(kMaxSmem)) P->nslot = ns;
    if (P->nslot < 2) return MLA_ERR_UNSUPPORTED;
    P->smem = decode_pair_smem_bytes(r, P->rope_half, P->nslot);
  } else {
    P->tmem_cols = pow2_at_least((2 + P->nch) * P->ncol, 32);
    if (P->tmem_cols > 512) return MLA_ERR_UNSUPPORTED;
    // Most cache slots that fit, preferring two P^T buffers; at least two slots.
    for (int npt = 2; npt >= 1 && P->nslot == 0; --npt) {
      for (int ns = kDecodeMaxSlots; ns >= 2; --ns) {
        if (decode_smem_bytes(P->ncol, P->nblk, P->slot_blocks, ns, npt) <= size_t(kMaxSmem)) {
          P->nslot = ns;
          P->npt = npt;
          break;
        }
      }
    }
    if (P->nslot < 2) return MLA_ERR_UNSUPPORTED;
    P->smem = decode_smem_bytes(P->ncol, P->nblk, P->slot_blocks, P->nslot, P->npt);
  }
  // Persistent grid: the units' page tiles are cut into `vgrid` equal ranges, one per CTA
  // (per cluster for the pair kernel). By default as many as fit on the device at once;
  // num_splits > 0 asks for num_splits ranges per unit on average.
  const int64_t max_tiles = (int64_t(max_seq_len) + kDecodeTok - 1) / kDecodeTok;
  // The range count is a multiple of the number of row blocks: range c works on row
  // block c % col_groups, so the blocks of a sequence are read in lockstep.
  const int cgs = P->col_groups;
  const int64_t resident = P->pair ? pair_clusters(P->smem) : num_sms();
  int64_t g = num_splits > 0 ? units * num_splits : resident;
  g = std::min<int64_t>(g, units * max_tiles);
  g = std::max<int64_t>(cgs, std::min<int64_t>(g, 1 << 20) / cgs * cgs);
  P->vgrid = int(g);
  P->grid = int(P->pair ? 2 * g : g);
  size_t off = 256;                              // device error word + padding
  P->range_off = off;                            // int32: tiles per range
  off += 256;
  P->unit_start_off = off;                       // int32 per unit: its first global tile
  off = align256(off + size_t(units) * sizeof(int32_t));
  P->part_lse_off = off;                         // two partial slots per range
  off = align256(off + size_t(g) * 2 * P->ncol * sizeof(float));
  P->part_o_off = off;                           // bf16: one rounding more than o_latent's
  off += size_t(g) * 2 * P->ncol * size_t(r) * sizeof(uint16_t);
  P->ws_bytes = off;
  return MLA_OK;
}

}  // namespace

extern "C" {

int32_t mla_row_width(const mla_dims* dims) {
  if (check_dims(dims) != MLA_OK) return -1;
  return row_width(dims);
}

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE_BOUNDS: return "MLA_ERR_DEVICE_BOUNDS";
    case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT";
  }
  return "MLA_ERR_UNKNOWN";
}

}  // extern "C"

namespace {

// Validation and parameters of mla_cache_append; *empty is set when there is nothing to do.
mla_status build_append(const mla_dims* dims, const void* c_kv, const void* k_r,
                        const float* rope_cos, const float* rope_sin, const int32_t* block_table,
                        int32_t max_pages_per_seq, const int32_t* start_pos, int32_t batch,
                        int32_t n_new, void* cache, int64_t num_pages, int32_t* dev_error,
                        AppendParams* out, bool* empty) {
  mla_status st = check_dims(dims);
  if (st != MLA_OK) return st;
  if (batch < 0 || n_new < 0 || max_pages_per_seq <= 0 || num_pages <= 0 ||
      num_pages > INT32_MAX)
    return MLA_ERR_INVALID_ARG;
  *empty = batch == 0 || n_new == 0;
  if (*empty) return MLA_OK;
  if (!c_kv || !block_table || !start_pos || !cache) return MLA_ERR_INVALID_ARG;
  if (dims->rope_dim > 0 && (!k_r || !rope_cos || !rope_sin)) return MLA_ERR_INVALID_ARG;
  if (!aligned(c_kv, 16) || !aligned(cache, 16)) return MLA_ERR_INVALID_ARG;
  AppendParams& p = *out;
  p = AppendParams{};
  p.c_kv = static_cast<const uint16_t*>(c_kv);
  p.k_r = static_cast<const uint16_t*>(k_r);
  p.rope_cos = rope_cos;
  p.rope_sin = rope_sin;
  p.block_table = block_table;
  p.start_pos = start_pos;
  p.cache = static_cast<uint16_t*>(cache);
  p.dev_error = dev_error;
  p.num_pages = num_pages;
  p.max_pages = max_pages_per_seq;
  p.batch = batch;
  p.n_new = n_new;
  p.r = dims->kv_lora_rank;
  p.groups = dims->num_kv_groups;
  p.rope_dim = dims->rope_dim;
  p.page_size = dims->page_size;
  return MLA_OK;
}

// The output tiles of absorb / out_up go out by TMA store when the strides allow it: box
// {128 features, 1 head, nr rows} over {M, H, rows}; columns past M and rows past `rows`
// are clipped by the TMA. Returns 0 (element copies) when the map cannot be made.
int encode_out_map(WGemmParams& p, void* out, int nr) {
  if (p.M % 8 != 0 || p.out_head_stride % 8 != 0 || p.out_row_stride % 8 != 0) return 0;
  const uint64_t d3[3] = {uint64_t(p.M), uint64_t(p.heads), uint64_t(p.rows)};
  const uint64_t s3[2] = {uint64_t(p.out_head_stride) * 2, uint64_t(p.out_row_stride) * 2};
  const uint32_t box[3] = {128, 1, uint32_t(nr)};
  return encode_bf16_map(&p.tm_out, out, 3, d3, s3, box, CU_TENSOR_MAP_SWIZZLE_NONE) ? 1 : 0;
}

static int pick_nr(int64_t rows) {
  return rows <= 16 ? 16 : rows <= 32 ? 32 : rows <= 64 ? 64 : 128;
}

// Validation and parameters of mla_absorb_q (tensor maps encoded); *nr is the row tile and
// *empty is set when there is nothing to do.
mla_status build_absorb(const mla_dims* dims, const void* q_nope, const void* q_pe,
                        const float* rope_cos, const float* rope_sin, const void* w_uk,
                        int64_t w_uk_head_stride, int32_t batch, int32_t q_len, void* q_ext,
                        WGemmParams* out, int* nr_out, bool* empty, bool encode = true) {
  mla_status st = check_dims(dims);
  if (st != MLA_OK) return st;
  if (batch < 0 || q_len <= 0) return MLA_ERR_INVALID_ARG;
  *empty = batch == 0;
  if (*empty) return MLA_OK;
  const int H = dims->num_heads, r = dims->kv_lora_rank, dn = dims->qk_nope_dim;
  if (!q_nope || !w_uk || !q_ext) return MLA_ERR_INVALID_ARG;
  if (dims->rope_dim > 0 && (!q_pe || !rope_cos || !rope_sin)) return MLA_ERR_INVALID_ARG;
  if (w_uk_head_stride < int64_t(dn) * r || w_uk_head_stride % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (!aligned(q_nope, 16) || !aligned(w_uk, 16) || !aligned(q_ext, 16)) return MLA_ERR_INVALID_ARG;
  const int64_t rows = int64_t(batch) * q_len;
  if (rows > int64_t(65535) * 128) return MLA_ERR_UNSUPPORTED;
  if (!encode) return MLA_OK;   // validation only
  const int D = row_width(dims);
  WGemmParams& p = *out;
  p = WGemmParams{};
  {
    const uint64_t dims3[3] = {uint64_t(r), uint64_t(dn), uint64_t(H)};
    const uint64_t str[2] = {uint64_t(r) * 2, uint64_t(w_uk_head_stride) * 2};
    const uint32_t box[3] = {64, 64, 1};
    if (!encode_bf16_map(&p.tm_w, w_uk, 3, dims3, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
  }
  const int nr = pick_nr(rows);
  {
    const uint64_t dims3[3] = {uint64_t(dn), uint64_t(H), uint64_t(rows)};
    const uint64_t str[2] = {uint64_t(dn) * 2, uint64_t(H) * dn * 2};
    const uint32_t box[3] = {64, 1, uint32_t(nr)};
    if (!encode_bf16_map(&p.tm_x, q_nope, 3, dims3, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
  }
  p.out = static_cast<uint16_t*>(q_ext);
  p.out_row_stride = int64_t(H) * D;
  p.out_head_stride = D;
  p.bias = nullptr;
  p.dev_error = nullptr;
  p.M = r;
  p.K = dn;
  p.rows = int32_t(rows);
  p.heads = H;
  p.a_mn = 1;
  p.q_pe = dims->rope_dim > 0 ? static_cast<const uint16_t*>(q_pe) : nullptr;
  p.rope_cos = rope_cos;
  p.rope_sin = rope_sin;
  p.groups = dims->num_kv_groups;
  p.rope_dim = dims->rope_dim;
  p.rope_vec = (dims->rope_dim % 8 == 0 && aligned(q_pe, 8) && aligned(rope_cos, 16) &&
                aligned(rope_sin, 16)) ? 1 : 0;
  p.tma_out = encode_out_map(p, p.out, nr);
  *nr_out = nr;
  return MLA_OK;
}

// Validation and parameters of mla_out_up (tensor maps encoded).
mla_status build_out_up(const mla_dims* dims, const void* o_latent, const void* w_uv,
                        int64_t w_uv_head_stride, const void* bias, int32_t rows, void* o,
                        WGemmParams* out, int* nr_out, bool* empty, bool encode = true) {
  mla_status st = check_dims(dims);
  if (st != MLA_OK) return st;
  if (rows < 0) return MLA_ERR_INVALID_ARG;
  *empty = rows == 0;
  if (*empty) return MLA_OK;
  const int H = dims->num_heads, r = dims->kv_lora_rank, dv = dims->v_head_dim;
  if (!o_latent || !w_uv || !o) return MLA_ERR_INVALID_ARG;
  if (w_uv_head_stride < int64_t(dv) * r || w_uv_head_stride % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (!aligned(o_latent, 16) || !aligned(w_uv, 16) || !aligned(o, 16)) return MLA_ERR_INVALID_ARG;
  if (int64_t(rows) > int64_t(65535) * 128) return MLA_ERR_UNSUPPORTED;
  if (!encode) return MLA_OK;   // validation only
  WGemmParams& p = *out;
  p = WGemmParams{};
  {
    const uint64_t dims3[3] = {uint64_t(r), uint64_t(dv), uint64_t(H)};
    const uint64_t str[2] = {uint64_t(r) * 2, uint64_t(w_uv_head_stride) * 2};
    const uint32_t box[3] = {64, 128, 1};
    if (!encode_bf16_map(&p.tm_w, w_uv, 3, dims3, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
  }
  const int nr = pick_nr(rows);
  {
    const uint64_t dims3[3] = {uint64_t(r), uint64_t(H), uint64_t(rows)};
    const uint64_t str[2] = {uint64_t(r) * 2, uint64_t(H) * r * 2};
    const uint32_t box[3] = {64, 1, uint32_t(nr)};
    if (!encode_bf16_map(&p.tm_x, o_latent, 3, dims3, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
  }
  p.out = static_cast<uint16_t*>(o);
  p.out_row_stride = int64_t(H) * dv;
  p.out_head_stride = dv;
  p.bias = static_cast<const uint16_t*>(bias);
  p.dev_error = nullptr;
  p.M = dv;
  p.K = r;
  p.rows = rows;
  p.heads = H;
  p.a_mn = 0;
  p.q_pe = nullptr;
  p.tma_out = encode_out_map(p, p.out, nr);
  *nr_out = nr;
  return MLA_OK;
}

}  // namespace

extern "C" {

mla_status mla_cache_append(const mla_dims* dims, const void* c_kv, const void* k_r,
                            const float* rope_cos, const float* rope_sin,
                            const int32_t* block_table, int32_t max_pages_per_seq,
                            const int32_t* start_pos, int32_t batch, int32_t n_new, void* cache,
                            int64_t num_pages, int32_t* dev_error, void* stream) {
  AppendParams p;
  bool empty = false;
  const mla_status st = build_append(dims, c_kv, k_r, rope_cos, rope_sin, block_table,
                                     max_pages_per_seq, start_pos, batch, n_new, cache,
                                     num_pages, dev_error, &p, &empty);
  if (st != MLA_OK || empty) return st;
  return launch_cache_append(p, as_stream(stream)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status mla_absorb_q(const mla_dims* dims, const void* q_nope, const void* q_pe,
                        const float* rope_cos, const float* rope_sin, const void* w_uk,
                        int64_t w_uk_head_stride, int32_t batch, int32_t q_len, void* q_ext,
                        void* stream) {
  WGemmParams p;
  int nr = 0;
  bool empty = false;
  const mla_status st = build_absorb(dims, q_nope, q_pe, rope_cos, rope_sin, w_uk,
                                     w_uk_head_stride, batch, q_len, q_ext, &p, &nr, &empty);
  if (st != MLA_OK || empty) return st;
  return launch_wgemm(p, nr, num_sms(), as_stream(stream)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status mla_out_up(const mla_dims* dims, const void* o_latent, const void* w_uv,
                      int64_t w_uv_head_stride, const void* bias, int32_t rows, void* o,
                      void* stream) {
  WGemmParams p;
  int nr = 0;
  bool empty = false;
  const mla_status st = build_out_up(dims, o_latent, w_uv, w_uv_head_stride, bias, rows, o, &p,
                                     &nr, &empty);
  if (st != MLA_OK || empty) return st;
  return launch_wgemm(p, nr, num_sms(), as_stream(stream)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status mla_down_kv_append(const mla_dims* dims, const void* hidden, int32_t hidden_dim,
                              const void* w_dkv, const float* rope_cos, const float* rope_sin,
                              const int32_t* block_table, int32_t max_pages_per_seq,
                              const int32_t* start_pos, int32_t batch, int32_t n_new, void* cache,
                              int64_t num_pages, int32_t* dev_error, void* kv_out, void* stream) {
  mla_status st = check_dims(dims);
  if (st != MLA_OK) return st;
  if (batch < 0 || n_new < 0 || hidden_dim <= 0 || hidden_dim % 8 != 0 ||
      max_pages_per_seq <= 0 || num_pages <= 0 || num_pages > INT32_MAX)
    return MLA_ERR_INVALID_ARG;
  if (batch == 0 || n_new == 0) return MLA_OK;
  const int r = dims->kv_lora_rank, R = dims->num_kv_groups * dims->rope_dim;
  if (!hidden || !w_dkv || !block_table || !start_pos || !cache) return MLA_ERR_INVALID_ARG;
  if (R > 0 && (!rope_cos || !rope_sin)) return MLA_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(w_dkv, 16) || !aligned(cache, 16) ||
      (kv_out && !aligned(kv_out, 16)))
    return MLA_ERR_INVALID_ARG;
  if (R > 128) return MLA_ERR_UNSUPPORTED;        // the rotary features share one tile
  const int64_t rows = int64_t(batch) * n_new;
  if (rows > INT32_MAX) return MLA_ERR_UNSUPPORTED;
  const int D = row_width(dims);
  const int nr = pick_nr(rows);
  DkvParams p{};
  {
    const uint64_t d2[2] = {uint64_t(hidden_dim), uint64_t(D)};
    const uint64_t s2[1] = {uint64_t(hidden_dim) * 2};
    const uint32_t box[2] = {64, 128};
    if (!encode_bf16_map(&p.tm_w, w_dkv, 2, d2, s2, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
  }
  {
    const uint64_t d2[2] = {uint64_t(hidden_dim), uint64_t(rows)};
    const uint64_t s2[1] = {uint64_t(hidden_dim) * 2};
    const uint32_t box[2] = {64, uint32_t(nr)};
    if (!encode_bf16_map(&p.tm_x, hidden, 2, d2, s2, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
  }
  p.cache = static_cast<uint16_t*>(cache);
  p.block_table = block_table;
  p.start_pos = start_pos;
  p.rope_cos = rope_cos;
  p.rope_sin = rope_sin;
  p.kv_out = static_cast<uint16_t*>(kv_out);
  p.dev_error = dev_error;
  p.num_pages = num_pages;
  p.max_pages = max_pages_per_seq;
  p.n_new = n_new;
  p.page_size = dims->page_size;
  p.r = r;
  p.groups = dims->num_kv_groups;
  p.rope_dim = dims->rope_dim;
  p.rows = int32_t(rows);
  p.K = hidden_dim;
  p.lat_tiles = (r + 127) / 128;
  p.n_nt = int32_t((rows + nr - 1) / nr);
  // the model width split across a cluster of up to 16 CTAs (the launcher lowers it to what
  // the device can co-schedule), at least 2 K blocks of 64 each
  const int nk = (hidden_dim + 63) / 64;
  p.splits = std::max(1, std::min(16, nk / 2));
  if (int64_t(p.lat_tiles + (R > 0 ? 1 : 0)) * p.n_nt * p.splits > (int64_t(1) << 31) - 1)
    return MLA_ERR_UNSUPPORTED;
  return launch_down_kv(p, nr, as_stream(stream)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // extern "C"

namespace {

// Workspace of mla_out_proj: counters, then the fp32 partials of stage B's K splits.
struct OProjPlan {
  int nr, n_nt, n_mt, splits, items, grid;
  size_t head_off, tile_off, part_off, bytes;
};

mla_status plan_oproj(const mla_dims* d, int32_t hidden, int32_t rows, OProjPlan* P) {
  mla_status st = check_dims(d);
  if (st != MLA_OK) return st;
  if (hidden <= 0 || hidden % 8 != 0 || rows < 0) return MLA_ERR_INVALID_ARG;
  if (d->v_head_dim % 64 != 0) return MLA_ERR_UNSUPPORTED;   // K splits on whole 64-blocks
  if (int64_t(rows) > int64_t(65535) * 128) return MLA_ERR_UNSUPPORTED;
  const int H = d->num_heads;
  P->nr = pick_nr(std::max(rows, 1));
  P->n_nt = (std::max(rows, 1) + P->nr - 1) / P->nr;
  P->n_mt = (hidden + 127) / 128;
  const int sms = num_sms();
  P->splits = std::max(1, std::min(H, sms / (P->n_mt * P->n_nt)));
  P->items = H * ((d->v_head_dim + 127) / 128) * P->n_nt + P->n_mt * P->splits * P->n_nt;
  P->grid = std::min(P->items, sms);
  size_t off = 256;                              // cta_done + padding
  P->head_off = off;
  off = align256(off + size_t(H) * 4);
  P->tile_off = off;
  off = align256(off + size_t(P->n_mt) * P->n_nt * 4);
  P->part_off = off;
  off += size_t(P->splits) * size_t(std::max(rows, 1)) * size_t(hidden) * 4;
  P->bytes = off;
  return MLA_OK;
}

}  // namespace

extern "C" {

size_t mla_out_proj_workspace_size(const mla_dims* dims, int32_t hidden, int32_t rows) {
  OProjPlan P;
  return plan_oproj(dims, hidden, rows, &P) == MLA_OK ? P.bytes : 0;
}

mla_status mla_out_proj(const mla_dims* dims, const void* o_latent, const void* w_uv,
                        int64_t w_uv_head_stride, const void* bias_v, const void* w_o,
                        const void* bias_o, int32_t hidden, int32_t rows, void* workspace,
                        size_t workspace_bytes, void* o, void* u, void* stream) {
  OProjPlan P;
  mla_status st = plan_oproj(dims, hidden, rows, &P);
  if (st != MLA_OK) return st;
  if (rows == 0) return MLA_OK;
  const int H = dims->num_heads, r = dims->kv_lora_rank, dv = dims->v_head_dim;
  if (!o_latent || !w_uv || !w_o || !o || !u) return MLA_ERR_INVALID_ARG;
  if (w_uv_head_stride < int64_t(dv) * r || w_uv_head_stride % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (!aligned(o_latent, 16) || !aligned(w_uv, 16) || !aligned(w_o, 16) || !aligned(o, 16) ||
      !aligned(u, 16))
    return MLA_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < P.bytes) return MLA_ERR_WORKSPACE;
  OProjParams p{};
  {
    const uint64_t d3[3] = {uint64_t(r), uint64_t(dv), uint64_t(H)};
    const uint64_t s3[2] = {uint64_t(r) * 2, uint64_t(w_uv_head_stride) * 2};
    const uint32_t box[3] = {64, 128, 1};
    if (!encode_bf16_map(&p.tm_wuv, w_uv, 3, d3, s3, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
  }
  {
    const uint64_t d3[3] = {uint64_t(r), uint64_t(H), uint64_t(rows)};
    const uint64_t s3[2] = {uint64_t(r) * 2, uint64_t(H) * r * 2};
    const uint32_t box[3] = {64, 1, uint32_t(P.nr)};
    if (!encode_bf16_map(&p.tm_ol, o_latent, 3, d3, s3, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
  }
  const uint64_t K = uint64_t(H) * dv;
  {
    const uint64_t d2[2] = {K, uint64_t(hidden)};
    const uint64_t s2[1] = {K * 2};
    const uint32_t box[2] = {64, 128};
    if (!encode_bf16_map(&p.tm_wo, w_o, 2, d2, s2, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
  }
  {
    const uint64_t d2[2] = {K, uint64_t(rows)};
    const uint64_t s2[1] = {K * 2};
    const uint32_t box[2] = {64, uint32_t(P.nr)};
    if (!encode_bf16_map(&p.tm_o, o, 2, d2, s2, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.o = static_cast<uint16_t*>(o);
  p.u = static_cast<uint16_t*>(u);
  p.bias_v = static_cast<const uint16_t*>(bias_v);
  p.bias_o = static_cast<const uint16_t*>(bias_o);
  p.part = reinterpret_cast<float*>(ws + P.part_off);
  p.head_done = reinterpret_cast<int32_t*>(ws + P.head_off);
  p.tile_done = reinterpret_cast<int32_t*>(ws + P.tile_off);
  p.cta_done = reinterpret_cast<int32_t*>(ws + 4);
  p.dev_error = reinterpret_cast<int32_t*>(ws);
  p.H = H;
  p.r = r;
  p.dv = dv;
  p.hidden = hidden;
  p.rows = rows;
  p.splits = P.splits;
  return launch_oproj(p, P.nr, P.grid, as_stream(stream)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

size_t mla_decode_workspace_size(const mla_dims* dims, int32_t batch, int32_t q_len,
                                 int32_t max_seq_len, int32_t num_splits) {
  DecodePlan P;
  if (plan_decode(dims, batch, q_len, max_seq_len, num_splits, &P) != MLA_OK) return 0;
  return P.ws_bytes;
}

}  // extern "C"

namespace {

// Validation, plan and parameters of mla_decode_attn (tensor maps encoded); *empty is set
// when there is nothing to do.
mla_status build_decode(const mla_dims* dims, const void* q_ext, const void* cache,
                        int64_t num_pages, const int32_t* block_table, int32_t max_pages_per_seq,
                        const int32_t* seq_lens, int32_t batch, int32_t q_len,
                        int32_t max_seq_len, int32_t causal, int32_t num_splits, void* workspace,
                        size_t workspace_bytes, void* o_latent, float* lse, DecodePlan* Pout,
                        DecodeParams* pout, bool* empty, bool encode = true) {
  DecodePlan& P = *Pout;
  mla_status st = plan_decode(dims, batch, q_len, max_seq_len, num_splits, &P);
  if (st != MLA_OK) return st;
  if (num_pages <= 0 || num_pages * kDecodeTok > (int64_t(1) << 31) || max_pages_per_seq <= 0 ||
      (causal != 0 && causal != 1))
    return MLA_ERR_INVALID_ARG;
  *empty = batch == 0;
  if (*empty) return MLA_OK;
  if (!q_ext || !cache || !block_table || !seq_lens || !o_latent || !lse)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(q_ext, 16) || !aligned(cache, 16)) return MLA_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256)) return MLA_ERR_WORKSPACE;
  if (workspace_bytes < P.ws_bytes) return MLA_ERR_WORKSPACE;
  if (!encode) return MLA_OK;   // validation only
  const int D = row_width(dims);
  const int64_t qH = int64_t(q_len) * dims->num_heads;
  DecodeParams& p = *pout;
  p = DecodeParams{};
  {
    const uint64_t d2[2] = {uint64_t(D), uint64_t(num_pages) * kDecodeTok};
    const uint64_t s2[1] = {uint64_t(D) * 2};
    const uint32_t box[2] = {64, uint32_t(kDecodeTok)};
    if (!encode_bf16_map(&p.tm_cache, cache, 2, d2, s2, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
  }
  {
    const uint64_t d3[3] = {uint64_t(D), uint64_t(qH), uint64_t(batch)};
    const uint64_t s3[2] = {uint64_t(D) * 2, uint64_t(qH) * D * 2};
    const uint32_t box[3] = {64, uint32_t(P.ncol), 1};
    if (!encode_bf16_map(&p.tm_q, q_ext, 3, d3, s3, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MLA_ERR_CUDA;
  }
  if (P.pair) {
    const uint64_t d2[2] = {uint64_t(D), uint64_t(num_pages) * kDecodeTok};
    const uint64_t s2[1] = {uint64_t(D) * 2};
    const uint32_t box[2] = {uint32_t(P.rope_half), uint32_t(kDecodeTok)};
    const CUtensorMapSwizzle sw = P.rope_half == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : P.rope_half == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                      : CU_TENSOR_MAP_SWIZZLE_32B;
    if (!encode_bf16_map(&p.tm_rope, cache, 2, d2, s2, box, sw)) return MLA_ERR_CUDA;
    p.q_ext = static_cast<const uint16_t*>(q_ext);
    p.rope_half = P.rope_half;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.o_latent = static_cast<uint16_t*>(o_latent);
  p.lse = lse;
  p.part_lse = reinterpret_cast<float*>(ws + P.part_lse_off);
  p.part_o = reinterpret_cast<uint16_t*>(ws + P.part_o_off);
  p.unit_start = reinterpret_cast<int32_t*>(ws + P.unit_start_off);
  p.range_len = reinterpret_cast<int32_t*>(ws + P.range_off);
  p.dev_error = reinterpret_cast<int32_t*>(ws);
  p.num_pages = num_pages;
  p.max_pages = max_pages_per_seq;
  p.batch = batch;
  p.q_len = q_len;
  p.num_heads = dims->num_heads;
  p.qH = int32_t(qH);
  p.r = dims->kv_lora_rank;
  p.D = D;
  p.nblk = P.nblk;
  p.nch = P.nch;
  p.col_groups = P.col_groups;
  p.units = P.units;
  p.max_seq_len = max_seq_len;
  p.causal = causal;
  p.nslot = P.nslot;
  p.slot_blocks = P.slot_blocks;
  p.tmem_cols = P.tmem_cols;
  p.npt = P.npt;
  p.scale_log2 = dims->softmax_scale * 1.4426950408889634f;
  return MLA_OK;
}

// The decode kernel of a built plan and, when units may be cut between CTAs, the merge (which
// then also brings `pf_bytes` at `pf`, the next kernel's weights, into L2; may be null).
mla_status launch_decode_plan(const DecodePlan& P, const DecodeParams& p, cudaStream_t s,
                              const void* pf = nullptr, int64_t pf_bytes = 0) {
  const cudaError_t le = P.pair ? launch_decode_pair(p, dim3(P.grid), P.smem, s)
                                : launch_decode(p, P.ncol, dim3(P.grid), P.smem, s);
  if (le != cudaSuccess) return MLA_ERR_CUDA;
  if (P.vgrid > P.col_groups) {
    // merge the pieces of units cut between CTAs (units held whole are skipped)
    CombineParams c{};
    c.part_o = p.part_o;
    c.part_lse = p.part_lse;
    c.unit_start = p.unit_start;
    c.range_len = p.range_len;
    c.seq_lens = p.seq_lens;
    c.o_latent = p.o_latent;
    c.lse = p.lse;
    c.q_len = p.q_len;
    c.max_seq_len = p.max_seq_len;
    c.max_pages = p.max_pages;
    c.qH = p.qH;
    c.r = p.r;
    c.ncol = P.ncol;
    c.col_groups = P.col_groups;
    c.units = P.units;
    c.vgrid = P.vgrid;
    c.sms = num_sms();
    c.l2_prefetch = pf;
    c.l2_prefetch_bytes = pf_bytes;
    if (launch_combine(c, s) != cudaSuccess) return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

}  // namespace

extern "C" {

mla_status mla_decode_attn(const mla_dims* dims, const void* q_ext, const void* cache,
                           int64_t num_pages, const int32_t* block_table,
                           int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                           int32_t q_len, int32_t max_seq_len, int32_t causal,
                           int32_t num_splits, void* workspace, size_t workspace_bytes,
                           void* o_latent, float* lse, void* stream) {
  DecodePlan P;
  DecodeParams p;
  bool empty = false;
  const mla_status st = build_decode(dims, q_ext, cache, num_pages, block_table,
                                     max_pages_per_seq, seq_lens, batch, q_len, max_seq_len,
                                     causal, num_splits, workspace, workspace_bytes, o_latent,
                                     lse, &P, &p, &empty);
  if (st != MLA_OK || empty) return st;
  return launch_decode_plan(P, p, as_stream(stream));
}

mla_status mla_decode_step(const mla_dims* dims, const void* c_kv_new, const void* k_r_new,
                           const float* rope_cos_new, const float* rope_sin_new,
                           const int32_t* start_pos, int32_t n_new, const void* q_nope,
                           const void* q_pe, const float* rope_cos_q, const float* rope_sin_q,
                           const void* w_uk, int64_t w_uk_head_stride, const void* w_uv,
                           int64_t w_uv_head_stride, const void* bias_v, void* cache,
                           int64_t num_pages, const int32_t* block_table,
                           int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                           int32_t q_len, int32_t max_seq_len, int32_t causal,
                           int32_t num_splits, void* q_ext, void* workspace,
                           size_t workspace_bytes, void* o_latent, float* lse, void* o,
                           void* stream) {
  // every part is validated (no tensor map encoded, nothing launched) before any is built
  AppendParams ap;
  bool ap_empty = false;
  mla_status st = build_append(dims, c_kv_new, k_r_new, rope_cos_new, rope_sin_new, block_table,
                               max_pages_per_seq, start_pos, batch, n_new, cache, num_pages,
                               static_cast<int32_t*>(workspace), &ap, &ap_empty);
  if (st != MLA_OK) return st;
  const int64_t rows = int64_t(batch) * q_len;
  if (rows > INT32_MAX) return MLA_ERR_UNSUPPORTED;
  WGemmParams ab, ou;
  DecodePlan P;
  DecodeParams dp;
  int nr_ab = 0, nr_ou = 0;
  bool ab_empty = false, de_empty = false, ou_empty = false;
  for (int pass = 0; pass < 2; ++pass) {
    const bool enc = pass == 1;
    st = build_absorb(dims, q_nope, q_pe, rope_cos_q, rope_sin_q, w_uk, w_uk_head_stride, batch,
                      q_len, q_ext, &ab, &nr_ab, &ab_empty, enc);
    if (st != MLA_OK) return st;
    st = build_decode(dims, q_ext, cache, num_pages, block_table, max_pages_per_seq, seq_lens,
                      batch, q_len, max_seq_len, causal, num_splits, workspace, workspace_bytes,
                      o_latent, lse, &P, &dp, &de_empty, enc);
    if (st != MLA_OK) return st;
    st = build_out_up(dims, o_latent, w_uv, w_uv_head_stride, bias_v, int32_t(rows), o, &ou,
                      &nr_ou, &ou_empty, enc);
    if (st != MLA_OK) return st;
    if (ab_empty) return MLA_OK;   // batch == 0: nothing to do anywhere
  }
  cudaStream_t s = as_stream(stream);
  if (!ap_empty) ab.app = ap;     // the absorption's epilogue warps write the new rows
  if (launch_wgemm(ab, nr_ab, num_sms(), s) != cudaSuccess) return MLA_ERR_CUDA;
  // the merge kernel (if the plan has one) brings W_UV into L2 for the up-projection
  st = launch_decode_plan(P, dp, s, w_uv, int64_t(dims->num_heads) * w_uv_head_stride * 2);
  if (st != MLA_OK) return st;
  return launch_wgemm(ou, nr_ou, num_sms(), s) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // extern "C"

namespace {

// The K = V form takes one key group, a query whose nope part is already in the latent
// space (d_n = r) and an output as wide as the cache row (d_v = r + d_r).
mla_status check_kv_shared(const mla_dims* d) {
  mla_status st = check_dims(d);
  if (st != MLA_OK) return st;
  if (d->num_kv_groups != 1 || d->rope_dim <= 0 || d->qk_nope_dim != d->kv_lora_rank ||
      d->v_head_dim != row_width(d))
    return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

mla_status kv_shared_rotate(const mla_dims* dims, const void* in, const float* rope_cos,
                            const float* rope_sin, int32_t batch, int32_t q_len, void* out,
                            int inverse, void* stream) {
  mla_status st = check_kv_shared(dims);
  if (st != MLA_OK) return st;
  if (batch < 0 || q_len <= 0) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (!in || !out || !rope_cos || !rope_sin) return MLA_ERR_INVALID_ARG;
  if (!aligned(in, 16) || !aligned(out, 16) || !aligned(rope_cos, 4) || !aligned(rope_sin, 4))
    return MLA_ERR_INVALID_ARG;
  KvSharedParams p{};
  p.in = static_cast<const uint16_t*>(in);
  p.out = static_cast<uint16_t*>(out);
  p.rope_cos = rope_cos;
  p.rope_sin = rope_sin;
  p.rows = int64_t(batch) * q_len * dims->num_heads;
  p.heads = dims->num_heads;
  p.r = dims->kv_lora_rank;
  p.rope_dim = dims->rope_dim;
  p.inverse = inverse;
  if (p.rows > (int64_t(1) << 36)) return MLA_ERR_UNSUPPORTED;
  return launch_kv_shared_rotate(p, as_stream(stream)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace

extern "C" {

mla_status mla_kv_shared_decode_dims(const mla_dims* dims, mla_dims* decode_dims) {
  mla_status st = check_kv_shared(dims);
  if (st != MLA_OK) return st;
  if (!decode_dims) return MLA_ERR_INVALID_ARG;
  const int32_t D = row_width(dims);
  *decode_dims = *dims;
  decode_dims->kv_lora_rank = D;
  decode_dims->qk_nope_dim = D;
  decode_dims->rope_dim = 0;
  decode_dims->v_head_dim = D;
  return MLA_OK;
}

mla_status mla_kv_shared_query(const mla_dims* dims, const void* q, const float* rope_cos,
                               const float* rope_sin, int32_t batch, int32_t q_len, void* q_ext,
                               void* stream) {
  return kv_shared_rotate(dims, q, rope_cos, rope_sin, batch, q_len, q_ext, 0, stream);
}

mla_status mla_kv_shared_output(const mla_dims* dims, const void* o_latent, const float* rope_cos,
                                const float* rope_sin, int32_t batch, int32_t q_len, void* o,
                                void* stream) {
  return kv_shared_rotate(dims, o_latent, rope_cos, rope_sin, batch, q_len, o, 1, stream);
}

mla_status mla_selftest_wait_timeout(int32_t* dev_error, void* stream) {
  if (!dev_error) return MLA_ERR_INVALID_ARG;
  mla_selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(dev_error);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status mla_get_device_status(const int32_t* dev_error, int32_t reset, void* stream) {
  if (!dev_error) return MLA_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, dev_error, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (reset) {
    if (cudaMemsetAsync(const_cast<int32_t*>(dev_error), 0, sizeof(int32_t), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return MLA_ERR_CUDA;
  }
  if (v & MLA_DEVERR_TIMEOUT) return MLA_ERR_DEVICE_TIMEOUT;
  if (v & MLA_DEVERR_BOUNDS) return MLA_ERR_DEVICE_BOUNDS;
  return MLA_OK;
}

}  // extern "C"
