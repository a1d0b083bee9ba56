// cg_common.cuh -- definitions shared by the libcachegen kernels and the C ABI.
//
// The container format and the arithmetic are specified in include/cachegen.h.
// This header only holds the constants, the section arithmetic and the small
// device helpers the encoder and decoder both use.
#pragma once

#include <cstdint>
#include <functional>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "cachegen.h"

namespace cg {

constexpr int kGroup = CG_GROUP;          // tokens per anchor group
constexpr uint32_t kProbBits = CG_PROB_BITS;
constexpr uint32_t kM = 1u << kProbBits;  // every frequency table sums to 4096
constexpr uint32_t kRansL = 1u << 15;     // lower bound of the 32-bit rANS state (x < 2^31)
constexpr int kAlphabet = 255;            // symbols u = v + 127 for v in [-127, 127]

// Limits of this implementation (checked by the C ABI before any launch).
constexpr int kMaxLayers = 1024;
constexpr int kMaxHeads = 64;
constexpr int kMaxHeadDim = 256;
constexpr int kMaxChunk = 16384;

struct Sections {
  uint64_t zp, scale, freq, offsets, payload;
};

__host__ __device__ inline uint64_t up16(uint64_t v) { return (v + 15) & ~uint64_t(15); }

// Byte offsets of the container sections for a chunk of n tokens.
__host__ __device__ inline Sections sections(int L, int H, int D, int64_t n) {
  const uint64_t chans = uint64_t(L) * 2 * H * D;
  Sections s;
  s.zp = CG_HEADER_BYTES;
  s.scale = up16(s.zp + 4 * chans);
  s.freq = up16(s.scale + 4 * chans);
  s.offsets = up16(s.freq + uint64_t(L) * 2 * H * 256 * 2);
  s.payload = up16(s.offsets + 4 * (uint64_t(L) * 2 * uint64_t(n) + 1));
  return s;
}

// Worst-case stream: one renormalisation word per symbol plus the two words of
// the flushed state.
__host__ __device__ inline uint64_t max_stream_bytes(int H, int D) {
  return 2 * (uint64_t(H) * D + 2);
}

// Per-stream scratch stride of the encoder (32-byte aligned so that 32-byte
// flushes stay aligned when written backwards from the region's end).
__host__ __device__ inline uint64_t scratch_stride(int H, int D) {
  return (max_stream_bytes(H, D) + 31) & ~uint64_t(31);
}

// Step of layer l at a level: [Practice] 3.1 prints the first / middle / last
// layer steps of the three levels; [Practice] 1 gives the shallow layers the
// finer step.  third(l) = floor(3l / L).
__host__ __device__ inline float step_of(int level, int l, int L) {
  const int third = (3 * l) / L;
  switch (level * 3 + third) {
    case 0: return 0.3f;
    case 1: return 0.8f;
    case 2: return 1.2f;
    case 3: return 0.5f;
    case 4: return 1.0f;
    case 5: return 1.5f;
    case 6: return 0.8f;
    case 7: return 1.5f;
    default: return 2.0f;
  }
}

// First error wins: the status word only changes from CG_OK.
__device__ __forceinline__ void set_status(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

// Workspace layout of the encoder, per call.
struct EncWorkspace {
  uint64_t sym;      // u8  [chunks][L][2][H][D/16][C][16]
  uint64_t etab;     // u32 [chunks][L][2][H][256][4]
  uint64_t lens;     // u32 [chunks][L][2][C]
  uint64_t slabtot;  // u32 [chunks][L][2]   words of each (layer, K/V)'s streams
  uint64_t scratch;  // u8  [chunks][L][2][C][scratch_stride]
  uint64_t total;
};

__host__ __device__ inline uint64_t up256(uint64_t v) { return (v + 255) & ~uint64_t(255); }

__host__ __device__ inline EncWorkspace enc_workspace(int L, int H, int D, int C, int chunks) {
  EncWorkspace w;
  const uint64_t streams = uint64_t(chunks) * L * 2 * C;
  w.sym = 0;
  w.etab = up256(w.sym + streams * uint64_t(H) * D);
  w.lens = up256(w.etab + uint64_t(chunks) * L * 2 * H * 256 * 16);
  w.slabtot = up256(w.lens + streams * 4);
  w.scratch = up256(w.slabtot + uint64_t(chunks) * L * 2 * 4);
  w.total = up256(w.scratch + streams * scratch_stride(H, D));
  return w;
}

// Workspace of the three-level encoder (cg_encode_levels): one encoder
// workspace whose stream lengths and word slots the three levels reuse in
// turn, plus a symbol array, constants and word totals for each level.
struct EncLevelsWorkspace {
  EncWorkspace base;  // level 0's symbols, constants and totals; shared lens and scratch
  uint64_t sym[3], etab[3], slabtot[3];
  uint64_t total;
};

__host__ __device__ inline EncLevelsWorkspace enc_levels_workspace(int L, int H, int D, int C,
                                                                   int chunks) {
  EncLevelsWorkspace w;
  w.base = enc_workspace(L, H, D, C, chunks);
  w.sym[0] = w.base.sym;
  w.etab[0] = w.base.etab;
  w.slabtot[0] = w.base.slabtot;
  const uint64_t streams = uint64_t(chunks) * L * 2 * C;
  uint64_t at = w.base.total;
  for (int k = 1; k < 3; ++k) {
    w.sym[k] = at;
    at = up256(at + streams * uint64_t(H) * D);
    w.etab[k] = at;
    at = up256(at + uint64_t(chunks) * L * 2 * H * 256 * 16);
    w.slabtot[k] = at;
    at = up256(at + uint64_t(chunks) * L * 2 * 4);
  }
  w.total = at;
  return w;
}

// Kernel launch parameters shared by the encoder kernels.
struct EncParams {
  const uint16_t* kv;      // [L][2][T][H][D]
  int64_t T;               // total tokens of kv
  int64_t token_start;     // first token of chunk 0
  int num_chunks;
  int C;                   // nominal chunk size
  int L, H, D;
  int level;
  int adjacent;            // 0: format 1 (deltas to the anchor); 1: format 2 (adjacent tokens)
  uint8_t* out;            // containers (null when only tables are built)
  uint64_t out_stride;
  uint64_t* out_sizes;     // [num_chunks]
  uint8_t* tables_out;     // table blocks written by cg_build_tables (or null)
  const uint8_t* tables_in;  // table blocks supplied to cg_encode (or null)
  uint64_t tables_stride;
  uint8_t* sym;            // workspace sections
  uint32_t* etab;
  uint32_t* lens;
  uint32_t* slabtot;
  uint8_t* scratch;
  int32_t* status;
  // Three-level encode only (quant_kernel<3>): per level, its symbols,
  // encoder constants, word totals and containers.
  uint8_t* lsym[3];
  uint32_t* letab[3];
  uint32_t* lslabtot[3];
  uint8_t* lout[3];
};

struct DecParams {
  const uint8_t* in;       // containers at in + k * in_stride
  uint64_t in_stride;
  int num_chunks;
  int C, L, H, D;
  int level;
  int adjacent;            // 1: format 2 containers (each delta against the previous token)
  uint16_t* out;
  uint64_t out_elems;      // size of out in elements (checked against the shape by the C ABI)
  int into;                // 0: chunk slots [L][2][n][H][D]; 1: full KV [L][2][T][H][D];
                           // 2: paged pool [L][2][num_pages][page_tokens][H][D]
  int64_t total_tokens;    // T of the full KV (modes 1 and 2)
  const int32_t* block_table;  // mode 2: physical page of logical page t / page_tokens
  int num_pages;           // mode 2
  int page_tokens;         // mode 2
  int units_per_slab;      // CTAs per (chunk, l, kv)
  int32_t* status;
};

// Id of the calling thread's current CUDA context; false when there is none
// (context.cu).
bool current_context_id(unsigned long long* id);

// Run first(stream) and second(side) with the device's side stream forked from
// `stream` before them and joined back into it after them (context.cu).  When
// no side stream can be had (no current context, resources not yet created
// during a graph capture, creation failed) nothing is queued, *forked stays
// false and the caller runs its work on `stream` alone.
cudaError_t fork_join(cudaStream_t stream, const std::function<cudaError_t(cudaStream_t)>& first,
                      const std::function<cudaError_t(cudaStream_t)>& second, bool* forked);

// Kernel launchers (encode.cu, decode.cu).
cudaError_t launch_encode(const EncParams& p, bool build_only, cudaStream_t stream);
cudaError_t launch_encode_levels(const EncParams& p, uint64_t* out_sizes, cudaStream_t stream);
cudaError_t launch_decode(const DecParams& p, cudaStream_t stream);

}  // namespace cg
