// capi.cu -- the extern "C" entry points of libcachegen (declared and
// documented in include/cachegen.h).  Argument checks happen here, on the
// host, before anything is enqueued; every device step is a kernel of
// encode.cu or decode.cu.
#include <cstdint>

#include "cg_common.cuh"

namespace cg {
int decode_units_per_slab(int C);
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cg_status check_shape(const cg_shape* s) {
  if (s == nullptr) return CG_ERR_INVALID_ARG;
  if (s->num_layers < 1 || s->num_kv_heads < 1 || s->head_dim < 1) return CG_ERR_INVALID_ARG;
  if (s->num_layers > cg::kMaxLayers || s->num_kv_heads > cg::kMaxHeads ||
      s->head_dim > cg::kMaxHeadDim || s->head_dim < 16 || (s->head_dim % 16) != 0)
    return CG_ERR_UNSUPPORTED;
  return CG_OK;
}

cg_status check_chunk(const cg_shape* s, int32_t chunk_tokens) {
  if (chunk_tokens < 1) return CG_ERR_INVALID_ARG;
  if (chunk_tokens > cg::kMaxChunk) return CG_ERR_UNSUPPORTED;
  // Every offset of the largest possible payload must fit in u32.
  const uint64_t worst = uint64_t(s->num_layers) * 2 * chunk_tokens *
                         cg::max_stream_bytes(s->num_kv_heads, s->head_dim);
  if (worst > 0xFFFFFFF0ull) return CG_ERR_UNSUPPORTED;
  return CG_OK;
}

bool valid_level(cg_level level) { return level >= CG_LEVEL_HIGH && level <= CG_LEVEL_FAST; }

// Common checks of the two encoder entry points.
cg_status check_encode_args(const cg_shape* shape, const uint16_t* kv_dev, int64_t total_tokens,
                            int64_t token_start, int32_t num_chunks, int32_t chunk_tokens,
                            cg_level level) {
  cg_status st = check_shape(shape);
  if (st != CG_OK) return st;
  if ((st = check_chunk(shape, chunk_tokens)) != CG_OK) return st;
  if (kv_dev == nullptr || !aligned16(kv_dev) || !valid_level(level)) return CG_ERR_INVALID_ARG;
  if (num_chunks < 1 || total_tokens < 1 || token_start < 0) return CG_ERR_INVALID_ARG;
  // Every chunk must hold at least one token.
  if (token_start + int64_t(num_chunks - 1) * chunk_tokens >= total_tokens)
    return CG_ERR_INVALID_ARG;
  if (uint64_t(num_chunks) * shape->num_layers * 2 * shape->num_kv_heads > 0x7FFFFFFFull ||
      uint64_t(num_chunks) * shape->num_layers * 2 * chunk_tokens > 0x7FFFFFFFull)
    return CG_ERR_UNSUPPORTED;
  return CG_OK;
}

cg_status check_decode_args(const cg_shape* shape, const uint8_t* in_dev, uint64_t in_stride,
                            int32_t num_chunks, int32_t chunk_tokens, cg_level level,
                            const uint16_t* out_dev, const int32_t* status_dev) {
  cg_status st = check_shape(shape);
  if (st != CG_OK) return st;
  if ((st = check_chunk(shape, chunk_tokens)) != CG_OK) return st;
  if (in_dev == nullptr || !aligned16(in_dev) || in_stride < CG_HEADER_BYTES ||
      (in_stride % 16) != 0 || num_chunks < 1 || !valid_level(level) || out_dev == nullptr ||
      !aligned16(out_dev) || status_dev == nullptr)
    return CG_ERR_INVALID_ARG;
  const uint64_t blocks = uint64_t(num_chunks) * shape->num_layers * 2 *
                          cg::decode_units_per_slab(chunk_tokens);
  if (blocks > 0x7FFFFFFFull) return CG_ERR_UNSUPPORTED;
  return CG_OK;
}

cg_status from_cuda(cudaError_t err) { return err == cudaSuccess ? CG_OK : CG_ERR_CUDA; }

}  // namespace

extern "C" {

const char* cg_status_string(cg_status status) {
  switch (status) {
    case CG_OK: return "ok";
    case CG_ERR_INVALID_ARG: return "invalid argument";
    case CG_ERR_CAPACITY: return "output or workspace too small";
    case CG_ERR_CORRUPT: return "corrupt container";
    case CG_ERR_MISMATCH: return "container or tables do not match the call";
    case CG_ERR_NONFINITE: return "non-finite input value";
    case CG_ERR_CUDA: return "CUDA error";
    case CG_ERR_UNSUPPORTED: return "shape outside the supported limits";
  }
  return "unknown status";
}

cg_status cg_section_offsets(const cg_shape* shape, int32_t n_tokens, uint64_t offs[5]) {
  cg_status st = check_shape(shape);
  if (st != CG_OK) return st;
  if (offs == nullptr || n_tokens < 1) return CG_ERR_INVALID_ARG;
  const cg::Sections s = cg::sections(shape->num_layers, shape->num_kv_heads, shape->head_dim,
                                      n_tokens);
  offs[0] = s.zp;
  offs[1] = s.scale;
  offs[2] = s.freq;
  offs[3] = s.offsets;
  offs[4] = s.payload;
  return CG_OK;
}

cg_status cg_encoded_bound(const cg_shape* shape, int32_t chunk_tokens, uint64_t* bytes) {
  cg_status st = check_shape(shape);
  if (st != CG_OK) return st;
  if ((st = check_chunk(shape, chunk_tokens)) != CG_OK) return st;
  if (bytes == nullptr) return CG_ERR_INVALID_ARG;
  const int L = shape->num_layers, H = shape->num_kv_heads, D = shape->head_dim;
  const cg::Sections s = cg::sections(L, H, D, chunk_tokens);
  *bytes = cg::up16(s.payload + uint64_t(L) * 2 * chunk_tokens * cg::max_stream_bytes(H, D));
  return CG_OK;
}

cg_status cg_tables_bytes(const cg_shape* shape, uint64_t* bytes) {
  cg_status st = check_shape(shape);
  if (st != CG_OK) return st;
  if (bytes == nullptr) return CG_ERR_INVALID_ARG;
  const int L = shape->num_layers, H = shape->num_kv_heads, D = shape->head_dim;
  const cg::Sections s = cg::sections(L, H, D, 1);
  *bytes = s.freq + uint64_t(L) * 2 * H * 512 - CG_HEADER_BYTES;
  return CG_OK;
}

cg_status cg_encode_workspace_bytes(const cg_shape* shape, int32_t chunk_tokens,
                                    int32_t num_chunks, uint64_t* bytes) {
  cg_status st = check_shape(shape);
  if (st != CG_OK) return st;
  if ((st = check_chunk(shape, chunk_tokens)) != CG_OK) return st;
  if (bytes == nullptr || num_chunks < 1) return CG_ERR_INVALID_ARG;
  *bytes = cg::enc_workspace(shape->num_layers, shape->num_kv_heads, shape->head_dim,
                             chunk_tokens, num_chunks)
               .total;
  return CG_OK;
}

cg_status cg_build_tables(const cg_shape* shape, const uint16_t* kv_dev, int64_t total_tokens,
                          int64_t token_start, int32_t num_chunks, int32_t chunk_tokens,
                          cg_level level, uint8_t* tables_dev, int32_t* status_dev,
                          void* workspace_dev, uint64_t workspace_bytes, cudaStream_t stream) {
  (void)workspace_dev;  // building tables needs no workspace
  (void)workspace_bytes;
  cg_status st =
      check_encode_args(shape, kv_dev, total_tokens, token_start, num_chunks, chunk_tokens, level);
  if (st != CG_OK) return st;
  if (tables_dev == nullptr || !aligned16(tables_dev) || status_dev == nullptr)
    return CG_ERR_INVALID_ARG;
  uint64_t tb = 0;
  cg_tables_bytes(shape, &tb);
  cg::EncParams p{};
  p.kv = kv_dev;
  p.T = total_tokens;
  p.token_start = token_start;
  p.num_chunks = num_chunks;
  p.C = chunk_tokens;
  p.L = shape->num_layers;
  p.H = shape->num_kv_heads;
  p.D = shape->head_dim;
  p.level = int(level);
  p.tables_out = tables_dev;
  p.tables_stride = tb;
  p.status = status_dev;
  return from_cuda(cg::launch_encode(p, true, stream));
}

static cg_status encode_common(const cg_shape* shape, const uint16_t* kv_dev,
                               int64_t total_tokens, int64_t token_start, int32_t num_chunks,
                               int32_t chunk_tokens, cg_level level, const uint8_t* tables_dev,
                               uint8_t* out_dev, uint64_t out_stride, uint64_t* out_sizes_dev,
                               int32_t* status_dev, void* workspace_dev,
                               uint64_t workspace_bytes, int adjacent, cudaStream_t stream) {
  cg_status st =
      check_encode_args(shape, kv_dev, total_tokens, token_start, num_chunks, chunk_tokens, level);
  if (st != CG_OK) return st;
  const int L = shape->num_layers, H = shape->num_kv_heads, D = shape->head_dim;
  if (out_dev == nullptr || !aligned16(out_dev) || out_sizes_dev == nullptr ||
      status_dev == nullptr || workspace_dev == nullptr || (out_stride % 16) != 0)
    return CG_ERR_INVALID_ARG;
  if (tables_dev != nullptr && !aligned16(tables_dev)) return CG_ERR_INVALID_ARG;
  // The header, table and offsets sections of a full chunk must fit; only the
  // data-dependent payload may overflow (reported through the status word).
  if (out_stride < cg::sections(L, H, D, chunk_tokens).payload) return CG_ERR_CAPACITY;
  const cg::EncWorkspace ws = cg::enc_workspace(L, H, D, chunk_tokens, num_chunks);
  if (workspace_bytes < ws.total || (reinterpret_cast<uintptr_t>(workspace_dev) & 255u) != 0)
    return workspace_bytes < ws.total ? CG_ERR_CAPACITY : CG_ERR_INVALID_ARG;
  uint64_t tb = 0;
  cg_tables_bytes(shape, &tb);
  uint8_t* w = static_cast<uint8_t*>(workspace_dev);
  cg::EncParams p{};
  p.kv = kv_dev;
  p.T = total_tokens;
  p.token_start = token_start;
  p.num_chunks = num_chunks;
  p.C = chunk_tokens;
  p.L = L;
  p.H = H;
  p.D = D;
  p.level = int(level);
  p.adjacent = adjacent;
  p.out = out_dev;
  p.out_stride = out_stride;
  p.out_sizes = out_sizes_dev;
  p.tables_in = tables_dev;
  p.tables_stride = tb;
  p.sym = w + ws.sym;
  p.etab = reinterpret_cast<uint32_t*>(w + ws.etab);
  p.lens = reinterpret_cast<uint32_t*>(w + ws.lens);
  p.slabtot = reinterpret_cast<uint32_t*>(w + ws.slabtot);
  p.scratch = w + ws.scratch;
  p.status = status_dev;
  return from_cuda(cg::launch_encode(p, false, stream));
}

cg_status cg_encode(const cg_shape* shape, const uint16_t* kv_dev, int64_t total_tokens,
                    int64_t token_start, int32_t num_chunks, int32_t chunk_tokens,
                    cg_level level, const uint8_t* tables_dev, uint8_t* out_dev,
                    uint64_t out_stride, uint64_t* out_sizes_dev, int32_t* status_dev,
                    void* workspace_dev, uint64_t workspace_bytes, cudaStream_t stream) {
  return encode_common(shape, kv_dev, total_tokens, token_start, num_chunks, chunk_tokens, level,
                       tables_dev, out_dev, out_stride, out_sizes_dev, status_dev, workspace_dev,
                       workspace_bytes, 0, stream);
}

cg_status cg_encode_adjacent(const cg_shape* shape, const uint16_t* kv_dev, int64_t total_tokens,
                             int64_t token_start, int32_t num_chunks, int32_t chunk_tokens,
                             cg_level level, uint8_t* out_dev, uint64_t out_stride,
                             uint64_t* out_sizes_dev, int32_t* status_dev, void* workspace_dev,
                             uint64_t workspace_bytes, cudaStream_t stream) {
  return encode_common(shape, kv_dev, total_tokens, token_start, num_chunks, chunk_tokens, level,
                       nullptr, out_dev, out_stride, out_sizes_dev, status_dev, workspace_dev,
                       workspace_bytes, 1, stream);
}

cg_status cg_encode_levels_workspace_bytes(const cg_shape* shape, int32_t chunk_tokens,
                                           int32_t num_chunks, uint64_t* bytes) {
  cg_status st = check_shape(shape);
  if (st != CG_OK) return st;
  if ((st = check_chunk(shape, chunk_tokens)) != CG_OK) return st;
  if (bytes == nullptr || num_chunks < 1) return CG_ERR_INVALID_ARG;
  *bytes = cg::enc_levels_workspace(shape->num_layers, shape->num_kv_heads, shape->head_dim,
                                    chunk_tokens, num_chunks)
               .total;
  return CG_OK;
}

cg_status cg_encode_levels(const cg_shape* shape, const uint16_t* kv_dev, int64_t total_tokens,
                           int64_t token_start, int32_t num_chunks, int32_t chunk_tokens,
                           uint8_t* out_dev, uint64_t out_stride, uint64_t* out_sizes_dev,
                           int32_t* status_dev, void* workspace_dev, uint64_t workspace_bytes,
                           cudaStream_t stream) {
  cg_status st = check_encode_args(shape, kv_dev, total_tokens, token_start, num_chunks,
                                   chunk_tokens, CG_LEVEL_BALANCED);
  if (st != CG_OK) return st;
  const int L = shape->num_layers, H = shape->num_kv_heads, D = shape->head_dim;
  if (out_dev == nullptr || !aligned16(out_dev) || out_sizes_dev == nullptr ||
      status_dev == nullptr || workspace_dev == nullptr || (out_stride % 16) != 0)
    return CG_ERR_INVALID_ARG;
  if (out_stride < cg::sections(L, H, D, chunk_tokens).payload) return CG_ERR_CAPACITY;
  const cg::EncLevelsWorkspace ws = cg::enc_levels_workspace(L, H, D, chunk_tokens, num_chunks);
  if (workspace_bytes < ws.total || (reinterpret_cast<uintptr_t>(workspace_dev) & 255u) != 0)
    return workspace_bytes < ws.total ? CG_ERR_CAPACITY : CG_ERR_INVALID_ARG;
  uint8_t* w = static_cast<uint8_t*>(workspace_dev);
  cg::EncParams p{};
  p.kv = kv_dev;
  p.T = total_tokens;
  p.token_start = token_start;
  p.num_chunks = num_chunks;
  p.C = chunk_tokens;
  p.L = L;
  p.H = H;
  p.D = D;
  p.level = CG_LEVEL_HIGH;
  p.out_stride = out_stride;
  p.lens = reinterpret_cast<uint32_t*>(w + ws.base.lens);
  p.scratch = w + ws.base.scratch;
  p.status = status_dev;
  for (int j = 0; j < 3; ++j) {
    p.lsym[j] = w + ws.sym[j];
    p.letab[j] = reinterpret_cast<uint32_t*>(w + ws.etab[j]);
    p.lslabtot[j] = reinterpret_cast<uint32_t*>(w + ws.slabtot[j]);
    p.lout[j] = out_dev + uint64_t(j) * num_chunks * out_stride;
  }
  return from_cuda(cg::launch_encode_levels(p, out_sizes_dev, stream));
}

static cg_status decode_common(const cg_shape* shape, const uint8_t* in_dev, uint64_t in_stride,
                               int32_t num_chunks, int32_t chunk_tokens, cg_level level,
                               uint16_t* out_dev, uint64_t out_elems, int into,
                               int64_t total_tokens, int32_t* status_dev, cudaStream_t stream,
                               const int32_t* block_table = nullptr, int32_t num_pages = 0,
                               int32_t page_tokens = 0, int adjacent = 0) {
  cg::DecParams p{};
  p.adjacent = adjacent;
  p.block_table = block_table;
  p.num_pages = num_pages;
  p.page_tokens = page_tokens;
  p.in = in_dev;
  p.in_stride = in_stride;
  p.num_chunks = num_chunks;
  p.C = chunk_tokens;
  p.L = shape->num_layers;
  p.H = shape->num_kv_heads;
  p.D = shape->head_dim;
  p.level = int(level);
  p.out = out_dev;
  p.out_elems = out_elems;
  p.into = into;
  p.total_tokens = total_tokens;
  p.units_per_slab = cg::decode_units_per_slab(chunk_tokens);
  p.status = status_dev;
  return from_cuda(cg::launch_decode(p, stream));
}

cg_status cg_decode(const cg_shape* shape, const uint8_t* in_dev, uint64_t in_stride,
                    int32_t num_chunks, int32_t chunk_tokens, cg_level level, uint16_t* out_dev,
                    uint64_t out_elems, int32_t* status_dev, cudaStream_t stream) {
  cg_status st = check_decode_args(shape, in_dev, in_stride, num_chunks, chunk_tokens, level,
                                   out_dev, status_dev);
  if (st != CG_OK) return st;
  const uint64_t slot = uint64_t(shape->num_layers) * 2 * chunk_tokens * shape->num_kv_heads *
                        shape->head_dim;
  if (out_elems < slot * uint64_t(num_chunks)) return CG_ERR_CAPACITY;
  return decode_common(shape, in_dev, in_stride, num_chunks, chunk_tokens, level, out_dev,
                       out_elems, 0, 0, status_dev, stream);
}

cg_status cg_decode_into(const cg_shape* shape, const uint8_t* in_dev, uint64_t in_stride,
                         int32_t num_chunks, int32_t chunk_tokens, cg_level level,
                         uint16_t* kv_dev, int64_t total_tokens, int32_t* status_dev,
                         cudaStream_t stream) {
  cg_status st = check_decode_args(shape, in_dev, in_stride, num_chunks, chunk_tokens, level,
                                   kv_dev, status_dev);
  if (st != CG_OK) return st;
  if (total_tokens < 1) return CG_ERR_INVALID_ARG;
  const uint64_t elems = uint64_t(shape->num_layers) * 2 * uint64_t(total_tokens) *
                         shape->num_kv_heads * shape->head_dim;
  return decode_common(shape, in_dev, in_stride, num_chunks, chunk_tokens, level, kv_dev, elems,
                       1, total_tokens, status_dev, stream);
}

cg_status cg_decode_adjacent(const cg_shape* shape, const uint8_t* in_dev, uint64_t in_stride,
                             int32_t num_chunks, int32_t chunk_tokens, cg_level level,
                             uint16_t* out_dev, uint64_t out_elems, int32_t* status_dev,
                             cudaStream_t stream) {
  cg_status st = check_decode_args(shape, in_dev, in_stride, num_chunks, chunk_tokens, level,
                                   out_dev, status_dev);
  if (st != CG_OK) return st;
  const uint64_t slot = uint64_t(shape->num_layers) * 2 * chunk_tokens * shape->num_kv_heads *
                        shape->head_dim;
  if (out_elems < slot * uint64_t(num_chunks)) return CG_ERR_CAPACITY;
  return decode_common(shape, in_dev, in_stride, num_chunks, chunk_tokens, level, out_dev,
                       out_elems, 0, 0, status_dev, stream, nullptr, 0, 0, 1);
}

cg_status cg_decode_adjacent_into(const cg_shape* shape, const uint8_t* in_dev,
                                  uint64_t in_stride, int32_t num_chunks, int32_t chunk_tokens,
                                  cg_level level, uint16_t* kv_dev, int64_t total_tokens,
                                  int32_t* status_dev, cudaStream_t stream) {
  cg_status st = check_decode_args(shape, in_dev, in_stride, num_chunks, chunk_tokens, level,
                                   kv_dev, status_dev);
  if (st != CG_OK) return st;
  if (total_tokens < 1) return CG_ERR_INVALID_ARG;
  const uint64_t elems = uint64_t(shape->num_layers) * 2 * uint64_t(total_tokens) *
                         shape->num_kv_heads * shape->head_dim;
  return decode_common(shape, in_dev, in_stride, num_chunks, chunk_tokens, level, kv_dev, elems,
                       1, total_tokens, status_dev, stream, nullptr, 0, 0, 1);
}

cg_status cg_decode_into_paged(const cg_shape* shape, const uint8_t* in_dev, uint64_t in_stride,
                               int32_t num_chunks, int32_t chunk_tokens, cg_level level,
                               uint16_t* pool_dev, int32_t num_pages, int32_t page_tokens,
                               const int32_t* block_table_dev, int64_t total_tokens,
                               int32_t* status_dev, cudaStream_t stream) {
  cg_status st = check_decode_args(shape, in_dev, in_stride, num_chunks, chunk_tokens, level,
                                   pool_dev, status_dev);
  if (st != CG_OK) return st;
  if (total_tokens < 1 || num_pages < 1 || page_tokens < 1 || block_table_dev == nullptr)
    return CG_ERR_INVALID_ARG;
  const uint64_t elems = uint64_t(shape->num_layers) * 2 * uint64_t(num_pages) *
                         uint64_t(page_tokens) * shape->num_kv_heads * shape->head_dim;
  return decode_common(shape, in_dev, in_stride, num_chunks, chunk_tokens, level, pool_dev,
                       elems, 2, total_tokens, status_dev, stream, block_table_dev, num_pages,
                       page_tokens);
}

cg_status cg_decode_adjacent_into_paged(const cg_shape* shape, const uint8_t* in_dev,
                                        uint64_t in_stride, int32_t num_chunks,
                                        int32_t chunk_tokens, cg_level level, uint16_t* pool_dev,
                                        int32_t num_pages, int32_t page_tokens,
                                        const int32_t* block_table_dev, int64_t total_tokens,
                                        int32_t* status_dev, cudaStream_t stream) {
  cg_status st = check_decode_args(shape, in_dev, in_stride, num_chunks, chunk_tokens, level,
                                   pool_dev, status_dev);
  if (st != CG_OK) return st;
  if (total_tokens < 1 || num_pages < 1 || page_tokens < 1 || block_table_dev == nullptr)
    return CG_ERR_INVALID_ARG;
  const uint64_t elems = uint64_t(shape->num_layers) * 2 * uint64_t(num_pages) *
                         uint64_t(page_tokens) * shape->num_kv_heads * shape->head_dim;
  return decode_common(shape, in_dev, in_stride, num_chunks, chunk_tokens, level, pool_dev,
                       elems, 2, total_tokens, status_dev, stream, block_table_dev, num_pages,
                       page_tokens, 1);
}

}  // extern "C"
