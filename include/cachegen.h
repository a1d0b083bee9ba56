/*
 * cachegen.h -- C ABI of libcachegen, a B200 (sm_100a) implementation of the
 * CacheGen KV-cache codec.
 *
 * What the codec computes.  Two pages are cited, by title and section:
 *   [Practice] "CacheGen实战：KV缓存压缩与流式传输在大型语言模型服务中的高效应用"
 *              (CacheGen in practice), sections 1 (why KV-cache compression
 *              helps), 2.1 (chunked pre-processing), 2.3 (parallel decode),
 *              3.1 (compression-level tuning);
 *   [Overview] "CacheGen：大语言模型推理加速的KV缓存压缩与流式传输技术解析"
 *              (CacheGen overview), sections "KV缓存的量化压缩机制" (KV-cache
 *              quantisation mechanism) and "量化编码器设计" (quantiser design).
 * Where the pages leave a step open, the plainest reading is fixed below.
 *
 *   - The KV cache is fp16, laid out [layer][K|V][token][kv_head][head_dim]
 *     (element (l, kv, t, h, d) at ((l*2 + kv)*T + t)*H*D + h*D + d).
 *     A *channel* is one (l, kv, h, d).
 *   - It is cut into chunks of C tokens ([Practice] 2.1 uses 1.5K = 1536); each
 *     chunk is encoded independently into one self-describing *container*.
 *   - Inside a chunk, tokens form groups of G = 10.  The first token of a
 *     group is its *anchor*, quantised to 8 bits per channel with a zero point
 *     and a scale taken from the range of the chunk's anchor tokens
 *     (per-channel scale and zero point: [Overview] KV-cache quantisation
 *     mechanism).
 *   - Every other token is stored as its difference to the *reconstructed*
 *     anchor of its group (delta coding of neighbouring tokens: [Practice] 1),
 *     quantised with a step that depends on which third of the layers it is
 *     in (shallow layers finer, deep layers coarser: [Practice] 1; the step
 *     tables: [Practice] 3.1):
 *                      first third  middle third  last third
 *        HIGH             0.3          0.8           1.2
 *        BALANCED         0.5          1.0           1.5
 *        FAST             0.8          1.5           2.0
 *     third(l) = floor(3*l / L).
 *   - Quantised symbols live in [-127, 127] and are entropy coded ("grouped
 *     entropy coding": [Practice] 1) with static rANS: one 12-bit
 *     frequency table per (layer, K/V, kv_head) built from the chunk's own
 *     histogram, one independent 32-bit rANS stream per (layer, K/V, token)
 *     holding that token's H*D symbols in [h][d] order, and an array of
 *     stream offsets.
 *   - Decode is the exact inverse (thread-parallel decode: [Practice]
 *     2.3) and rebuilds fp16 values as fp16_rn(a + (float)q * s) with both
 *     operations rounded to nearest and no fused multiply-add.
 *
 * Exact arithmetic (everything fp32, IEEE round-to-nearest-even, no FMA):
 *   anchor range per channel over local tokens 0, 10, 20, ... of the chunk:
 *       lo = min, hi = max;  zp = (lo + hi) * 0.5f;  scale = (hi - lo) / 254.0f
 *   anchor code  c = scale == 0 ? 0 : clamp(roundf((x - zp) / scale), -127, 127)
 *   anchor value a = zp + (float)c * scale
 *   delta code   q = clamp(roundf((x - a_group) / step), -127, 127)
 *   delta value      a_group + (float)q * step
 *   roundf rounds half away from zero.  Output is fp16 round-to-nearest-even.
 *
 * Frequency table of one (l, kv, h) over N = n*D symbols, symbol index
 * u = v + 127 in [0, 254] (slot 255 is always 0):
 *   f[u] = count[u] ? max(1, floor(count[u] * 4096 / N)) : 0
 *   if sum f < 4096: the symbol with the largest count (ties: smallest u)
 *                    receives 4096 - sum f
 *   while sum f > 4096: among u with f[u] > 1, the largest f (ties: smallest
 *                    u) is decremented by one
 *   cum[u] = sum of f[u'] for u' < u.
 *
 * rANS (32-bit state x in [2^15, 2^31), 16-bit words, 12-bit probabilities):
 *   encode symbols j = H*D-1 down to 0 starting from x = 2^15:
 *       if x >= f << 19: emit x & 0xFFFF, x >>= 16
 *       x = (x / f) * 4096 + x % f + cum
 *   then emit x & 0xFFFF and x >> 16.  The stream is the emitted words in
 *   reverse order, little-endian u16.  Decode reads x = (w0 << 16) | w1, then
 *   per symbol: slot = x & 4095, u = the symbol with cum[u] <= slot <
 *   cum[u] + f[u], x = f * (x >> 12) + slot - cum, and if x < 2^15 then
 *   x = (x << 16) | next word.  A valid stream ends with x == 2^15 and every
 *   word consumed.
 *
 * Container (one per chunk, little-endian, every section starts on a 16-byte
 * boundary, padding bytes are zero):
 *   [0, 64)  header (cg_header below)
 *   zp      f32 [L][2][H][D]
 *   scale   f32 [L][2][H][D]
 *   freq    u16 [L][2][H][256]
 *   offsets u32 [2*L*n + 1]   byte offset of stream (l, kv, t) -- index
 *                             (l*2 + kv)*n + t -- from the payload start;
 *                             the last entry is the payload size
 *   payload the streams back to back
 *   total_bytes = round_up(payload offset + payload bytes, 16)
 *
 * Conventions of every call below:
 *   - Pointers named *_dev are device memory; everything else is host memory.
 *     The caller owns and allocates every buffer; no call allocates device
 *     memory, frees or synchronises.  All device work is ordered on `stream`
 *     (0 = legacy default stream) and the calls return before it completes.
 *     cg_encode and cg_encode_adjacent run the second half of a call of two
 *     or more chunks on a library-owned stream, forked from `stream` by an
 *     event before it and joined back into `stream` after it, so work queued
 *     on `stream` later still sees the whole call done (under graph capture
 *     the pair is captured as a fork and a join).  That stream and its two
 *     events are created on the first such call per device and context; a
 *     call made while `stream` is being captured before they exist runs on
 *     `stream` alone.  Calls on different streams share the library stream,
 *     so their second halves run one after the other.
 *   - fp16 values are passed as their uint16_t bit patterns.
 *   - Argument, shape and size errors are returned synchronously and nothing
 *     is enqueued.  Data-dependent errors (corrupt container, non-finite
 *     input, header mismatch, capacity) are written by the kernels to
 *     *status_dev with "first error wins" (an atomic compare-and-swap from
 *     CG_OK); the library never resets it, so the caller zeroes it before the
 *     first call and reads it after synchronising.  CG_ERR_CUDA is returned
 *     when a launch fails.
 *   - Shape limits: 1 <= L <= 1024, 1 <= H <= 64, 16 <= D <= 256 with
 *     D % 16 == 0, 1 <= chunk_tokens <= 16384, and the worst-case payload of
 *     one chunk must fit the u32 offsets (cg_encoded_bound checks this).
 *   - Device buffers holding fp16 or containers must be 16-byte aligned, and
 *     container strides multiples of 16.
 */
#ifndef CACHEGEN_H_
#define CACHEGEN_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CG_FORMAT_VERSION 1          /* deltas to the group's reconstructed anchor */
#define CG_FORMAT_VERSION_ADJACENT 2 /* deltas to the previous token (cg_encode_adjacent) */
#define CG_MAGIC 0x314B4743u /* bytes "CGK1" */
#define CG_GROUP 10
#define CG_PROB_BITS 12
#define CG_HEADER_BYTES 64

typedef enum cg_level {
  CG_LEVEL_HIGH = 0,     /* steps 0.3 / 0.8 / 1.2 */
  CG_LEVEL_BALANCED = 1, /* steps 0.5 / 1.0 / 1.5 */
  CG_LEVEL_FAST = 2      /* steps 0.8 / 1.5 / 2.0 */
} cg_level;

typedef enum cg_status {
  CG_OK = 0,
  CG_ERR_INVALID_ARG = 1, /* bad pointer, size, level or shape (synchronous) */
  CG_ERR_CAPACITY = 2,    /* output or workspace too small */
  CG_ERR_CORRUPT = 3,     /* container malformed or a stream does not decode cleanly */
  CG_ERR_MISMATCH = 4,    /* header disagrees with the call (level, chunk size, shape,
                             token range), or supplied tables lack a symbol */
  CG_ERR_NONFINITE = 5,   /* the fp16 input holds a NaN or an infinity */
  CG_ERR_CUDA = 6,        /* a CUDA launch or runtime call failed */
  CG_ERR_UNSUPPORTED = 7  /* shape outside the limits listed above */
} cg_status;

typedef struct cg_shape {
  int32_t num_layers;   /* L */
  int32_t num_kv_heads; /* H */
  int32_t head_dim;     /* D */
} cg_shape;

/* The 64-byte container header, exactly as stored. */
typedef struct cg_header {
  uint32_t magic;         /* CG_MAGIC */
  uint16_t version;       /* CG_FORMAT_VERSION, or CG_FORMAT_VERSION_ADJACENT (format 2) */
  uint8_t level;          /* cg_level */
  uint8_t group;          /* CG_GROUP */
  uint32_t num_layers;    /* L */
  uint32_t num_kv_heads;  /* H */
  uint32_t head_dim;      /* D */
  uint32_t chunk_tokens;  /* nominal chunk size C */
  uint32_t n_tokens;      /* tokens in this chunk, 1..C */
  uint32_t prob_bits;     /* CG_PROB_BITS */
  uint64_t token_start;   /* first token of the chunk in the full sequence */
  uint64_t payload_bytes; /* size of the payload section */
  uint64_t total_bytes;   /* size of the whole container */
  uint64_t reserved;      /* 0 */
} cg_header;

/* Human-readable name of a status code (static string, never NULL). */
const char* cg_status_string(cg_status status);

/* Byte offset of each container section for a chunk of n tokens.  Host, pure.
 * offs[0..4] = zp, scale, freq, offsets, payload. */
cg_status cg_section_offsets(const cg_shape* shape, int32_t n_tokens, uint64_t offs[5]);

/* Largest container a chunk of `chunk_tokens` tokens can produce (every symbol
 * costing one 16-bit renormalisation word).  A container slot of this size
 * never overflows.  Host, pure. */
cg_status cg_encoded_bound(const cg_shape* shape, int32_t chunk_tokens, uint64_t* bytes);

/* Size of the per-chunk table block written by cg_build_tables: the zp, scale
 * and freq sections of a container, laid out as in the container
 * (offsets measured from the block start = container offset 64).  Host, pure. */
cg_status cg_tables_bytes(const cg_shape* shape, uint64_t* bytes);

/* Device workspace cg_encode and cg_build_tables need for `num_chunks` chunks
 * of `chunk_tokens`.  Host, pure. */
cg_status cg_encode_workspace_bytes(const cg_shape* shape, int32_t chunk_tokens,
                                    int32_t num_chunks, uint64_t* bytes);

/* Build the quantiser parameters and frequency tables of `num_chunks`
 * consecutive chunks.  Chunk k covers tokens [token_start + k*C,
 * min(token_start + (k+1)*C, total_tokens)) of kv_dev ([L][2][total_tokens][H][D]
 * fp16); every chunk must hold at least one token.  tables_dev receives
 * num_chunks blocks of cg_tables_bytes each, at that stride.  Grounding: the
 * per-chunk pre-processing of [Practice] 2.1 and the per-channel parameters
 * of [Overview] KV-cache quantisation mechanism.
 * Data errors: CG_ERR_NONFINITE. */
cg_status cg_build_tables(const cg_shape* shape, const uint16_t* kv_dev, int64_t total_tokens,
                          int64_t token_start, int32_t num_chunks, int32_t chunk_tokens,
                          cg_level level, uint8_t* tables_dev, int32_t* status_dev,
                          void* workspace_dev, uint64_t workspace_bytes, cudaStream_t stream);

/* Encode `num_chunks` consecutive chunks (same token ranges as
 * cg_build_tables) at `level`.  Container k is written to out_dev + k*out_stride
 * and its size to out_sizes_dev[k] (u64, device).  tables_dev == NULL builds
 * the tables from the data (the normal path); otherwise the blocks of a
 * previous cg_build_tables call are used as they are.  A container that does
 * not fit out_stride sets CG_ERR_CAPACITY, stores the required size in
 * out_sizes_dev[k] and leaves the slot's payload unwritten; out_stride >=
 * cg_encoded_bound never overflows.  Grounding: [Practice] 1, 2.1
 * and 3.1; [Overview] quantiser design.  Data errors: CG_ERR_NONFINITE, CG_ERR_CAPACITY, CG_ERR_MISMATCH
 * (supplied tables give a used symbol frequency 0). */
cg_status cg_encode(const cg_shape* shape, const uint16_t* kv_dev, int64_t total_tokens,
                    int64_t token_start, int32_t num_chunks, int32_t chunk_tokens,
                    cg_level level, const uint8_t* tables_dev, uint8_t* out_dev,
                    uint64_t out_stride, uint64_t* out_sizes_dev, int32_t* status_dev,
                    void* workspace_dev, uint64_t workspace_bytes, cudaStream_t stream);

/* Decode `num_chunks` containers, container k at in_dev + k*in_stride (at most
 * in_stride bytes are read from it).  Chunk k's values go to
 * out_dev + k*(L*2*chunk_tokens*H*D) laid out [L][2][n_k][H][D], n_k from its
 * header; out_elems is the size of out_dev in elements.  Each header must
 * carry this call's shape, level and chunk size (else CG_ERR_MISMATCH).
 * Grounding: [Practice] 2.3 (the decode thread).  Data errors:
 * CG_ERR_CORRUPT, CG_ERR_MISMATCH.  No workspace: all staging is on chip. */
cg_status cg_decode(const cg_shape* shape, const uint8_t* in_dev, uint64_t in_stride,
                    int32_t num_chunks, int32_t chunk_tokens, cg_level level, uint16_t* out_dev,
                    uint64_t out_elems, int32_t* status_dev, cudaStream_t stream);

/* As cg_decode, but each chunk is written into the full KV buffer kv_dev
 * ([L][2][total_tokens][H][D]) at the token_start stored in its header, which
 * must satisfy token_start + n <= total_tokens (else CG_ERR_MISMATCH).
 * Grounding: [Practice] 2.3 (the fill thread that injects decoded KV into
 * the model). */
cg_status cg_decode_into(const cg_shape* shape, const uint8_t* in_dev, uint64_t in_stride,
                         int32_t num_chunks, int32_t chunk_tokens, cg_level level,
                         uint16_t* kv_dev, int64_t total_tokens, int32_t* status_dev,
                         cudaStream_t stream);

/* As cg_decode_into, but into a paged KV pool, the layout of serving engines
 * that hand out the cache in fixed-size token pages through a block table.
 * pool_dev holds num_pages pages of page_tokens tokens for every (layer, K/V):
 * [L][2][num_pages][page_tokens][H][D] (16-byte aligned).  Logical token t
 * (0 <= t < total_tokens, the sequence's capacity) lives in row
 * t % page_tokens of page block_table_dev[t / page_tokens]; block_table_dev
 * (int32, device, read only) has ceil(total_tokens / page_tokens) entries.
 * Each chunk lands at the token_start stored in its header, which must satisfy
 * token_start + n <= total_tokens (else CG_ERR_MISMATCH).  A block-table entry
 * outside [0, num_pages) sets CG_ERR_MISMATCH and nothing is written for the
 * tokens of that page.  Grounding: [Practice] 2.3 (the fill thread that
 * injects decoded KV into the model's cache); the page layout is the
 * integration this call serves, the pages do not fix it. */
cg_status cg_decode_into_paged(const cg_shape* shape, const uint8_t* in_dev, uint64_t in_stride,
                               int32_t num_chunks, int32_t chunk_tokens, cg_level level,
                               uint16_t* pool_dev, int32_t num_pages, int32_t page_tokens,
                               const int32_t* block_table_dev, int64_t total_tokens,
                               int32_t* status_dev, cudaStream_t stream);

/* Format 2: deltas between adjacent tokens.  [Practice] 1 describes the
 * deltas as differences between adjacent tokens; format 1 (every call above)
 * takes them against the group's reconstructed anchor so that every token
 * decodes on its own.  Format 2 takes the page literally: inside a group,
 * token t is quantised against the reconstruction of token t - 1,
 *     q_t = clamp(roundf((x_t - x^_(t-1)) / step), -127, 127),
 *     x^_t = x^_(t-1) + (float)q_t * step      (x^ of the anchor = a),
 * each operation fp32 and rounded to nearest, no fused multiply-add; the chain
 * restarts at every anchor, so a value depends on at most nine earlier ones.
 * Anchors, tables, streams and the container layout are those of format 1;
 * the header's version field is CG_FORMAT_VERSION_ADJACENT.  A format-2
 * container given to a format-1 decoder, or the other way round, is
 * CG_ERR_MISMATCH. */

/* cg_encode writing format 2.  Arguments as cg_encode without tables_dev (the
 * tables are always built from the format-2 symbols); the workspace is
 * cg_encode_workspace_bytes. */
cg_status cg_encode_adjacent(const cg_shape* shape, const uint16_t* kv_dev, int64_t total_tokens,
                             int64_t token_start, int32_t num_chunks, int32_t chunk_tokens,
                             cg_level level, uint8_t* out_dev, uint64_t out_stride,
                             uint64_t* out_sizes_dev, int32_t* status_dev, void* workspace_dev,
                             uint64_t workspace_bytes, cudaStream_t stream);

/* cg_decode of format-2 containers (same arguments and layout).  The decoder
 * rebuilds each group's chain from its anchor in the same pass that decodes
 * the streams.  As in every decode call, a slot whose chunk or stream is
 * reported corrupt holds undefined values. */
cg_status cg_decode_adjacent(const cg_shape* shape, const uint8_t* in_dev, uint64_t in_stride,
                             int32_t num_chunks, int32_t chunk_tokens, cg_level level,
                             uint16_t* out_dev, uint64_t out_elems, int32_t* status_dev,
                             cudaStream_t stream);

/* cg_decode_into of format-2 containers (same arguments). */
cg_status cg_decode_adjacent_into(const cg_shape* shape, const uint8_t* in_dev,
                                  uint64_t in_stride, int32_t num_chunks, int32_t chunk_tokens,
                                  cg_level level, uint16_t* kv_dev, int64_t total_tokens,
                                  int32_t* status_dev, cudaStream_t stream);

/* cg_decode_into_paged of format-2 containers (same arguments and pool
 * layout).  A token whose page is unmapped is not written and sets
 * CG_ERR_MISMATCH; the later tokens of its group are still written, because
 * each group's chain is rebuilt from the decoded values, never read back from
 * the pool. */
cg_status cg_decode_adjacent_into_paged(const cg_shape* shape, const uint8_t* in_dev,
                                        uint64_t in_stride, int32_t num_chunks,
                                        int32_t chunk_tokens, cg_level level, uint16_t* pool_dev,
                                        int32_t num_pages, int32_t page_tokens,
                                        const int32_t* block_table_dev, int64_t total_tokens,
                                        int32_t* status_dev, cudaStream_t stream);

/* Device workspace cg_encode_levels needs for `num_chunks` chunks of
 * `chunk_tokens` (about three times the symbol part of cg_encode's).  Host,
 * pure. */
cg_status cg_encode_levels_workspace_bytes(const cg_shape* shape, int32_t chunk_tokens,
                                           int32_t num_chunks, uint64_t* bytes);

/* Encode `num_chunks` consecutive chunks (the token ranges of cg_encode) at
 * all three levels from one read of the fp16 cache.  Grounding: [Practice]
 * 2.1 prepares three versions of every chunk ahead of sending, so that the
 * sender can choose one per chunk as the bandwidth changes ([Practice] 2.2).
 * The anchor range, the anchor codes and the reconstructed anchors do not
 * depend on the level and are computed once; every delta is quantised at the
 * three levels' steps in the same pass, and each level's histograms, tables
 * and streams are then built as in cg_encode.
 * Output: the container of (level j, chunk k) -- j = CG_LEVEL_HIGH,
 * CG_LEVEL_BALANCED, CG_LEVEL_FAST -- goes to
 * out_dev + (j*num_chunks + k)*out_stride and its size to
 * out_sizes_dev[j*num_chunks + k] (u64, device); it is byte for byte the
 * container cg_encode writes for that chunk at level j.  Tables are always
 * built from the data.  The workspace (cg_encode_levels_workspace_bytes,
 * 256-byte aligned) is the caller's, as for cg_encode.  Data errors:
 * CG_ERR_NONFINITE, CG_ERR_CAPACITY (per container, as cg_encode). */
cg_status cg_encode_levels(const cg_shape* shape, const uint16_t* kv_dev, int64_t total_tokens,
                           int64_t token_start, int32_t num_chunks, int32_t chunk_tokens,
                           uint8_t* out_dev, uint64_t out_stride, uint64_t* out_sizes_dev,
                           int32_t* status_dev, void* workspace_dev, uint64_t workspace_bytes,
                           cudaStream_t stream);

/* cg_encode without caller-provided scratch.  The pages have no counterpart
 * to this call; it exists for callers that cannot allocate device memory --
 * an inference server that has reserved the whole GPU for its own pool, a
 * plugin whose enqueue step must not call cudaMalloc, or a latency-critical
 * path that cannot take an allocation's implicit synchronisation.  Arguments
 * and results are those of cg_encode minus the workspace pair.  The scratch is
 * one fixed 128 MiB block of device memory inside the library, reserved on
 * every GPU that loads the library and held until the process exits; calls
 * whose cg_encode_workspace_bytes exceeds 128 MiB return CG_ERR_CAPACITY.  The
 * first call on a device looks up the block's device address (a host-side
 * query), and so does the first call after the device's context was destroyed
 * and created again (cudaDeviceReset); make that first call before any stream
 * capture.  Every call uses
 * the same block, so calls that overlap on the GPU (other streams, other
 * host threads) race and must be serialised by the caller.  Nothing in the
 * block needs clearing: each call writes every byte it reads.  No allocation
 * of any kind happens in this call. */
cg_status cg_encode_static(const cg_shape* shape, const uint16_t* kv_dev, int64_t total_tokens,
                           int64_t token_start, int32_t num_chunks, int32_t chunk_tokens,
                           cg_level level, const uint8_t* tables_dev, uint8_t* out_dev,
                           uint64_t out_stride, uint64_t* out_sizes_dev, int32_t* status_dev,
                           cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CACHEGEN_H_ */
