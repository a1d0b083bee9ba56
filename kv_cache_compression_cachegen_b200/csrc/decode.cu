// decode.cu -- fused rANS decode -> dequantise -> fp16 store (cg_decode,
// cg_decode_into, cg_decode_into_paged), and the two-pass decode of format 2
// (cg_decode_adjacent, cg_decode_adjacent_into: decode_kernel<true> stores the
// symbols, chain_kernel rebuilds the adjacent-token chains; see chain_kernel).
//
// [Practice] 2.3 (parallel decode): the receiver decodes on the GPU with one
// thread per token and hands the result to the thread that fills the model's
// KV cache.  Here one thread owns one rANS stream, i.e. one (layer, K/V,
// token), and writes its fp16 values straight into the destination layout, so
// decode and fill are one kernel.
//
// CTA = one "unit": 32 anchor groups (320 tokens) of one (chunk, layer, K/V).
//   warp 0      decodes the 32 anchor streams (lane g -> token 10 g);
//   warps 1..9  decode the 288 delta streams (9 per group).
// Every stream holds H*D symbols in [h][d] order and every head has its own
// frequency table, so the CTA walks the heads in lockstep:
//   iteration it:  anchor warp decodes head it      with table it % 3,
//                  delta warps decode head it - 1   with table (it-1) % 3,
//                  all threads fill the slot table of head it + 1,
//                  one warp scans the frequencies of head it + 2.
// The anchor warp runs one head ahead so that the reconstructed anchors a_g of
// head it-1 (fp32, in shared memory) are ready when the delta warps need them;
// one __syncthreads per head separates the iterations.
//
// Compressed words reach a thread through a 64-byte ring in shared memory
// (four 16-byte blocks, plus a copy of the first block after the last, so that
// the reads of one step never wrap).  Every 8 symbols the thread issues at most one
// cp.async for the next block of its stream and waits only for the blocks
// issued two steps earlier; since 8 symbols consume at most 8 words (one
// block), the words a step can read were always requested at least two steps
// before, so global-memory latency stays off the decode chain.
//
// Per symbol: one slot-table lookup, the state update, an optional 16-bit
// refill from the ring, and the dequantisation a + (float)q * s with IEEE
// round-to-nearest adds and multiplies (no contraction).  The slot entry keeps
// the symbol in its top byte, so (float)q comes from a byte permute and one
// exact subtraction instead of a second shared-memory lookup.
//
// Output: a thread's values of two steps (16 fp16, 32 contiguous bytes of its
// token's row) leave as one 256-bit store, a full L2 sector.  Every thread
// writes its own row, so a warp's store touches 32 rows; with 16-byte stores
// the L2 had to take twice as many partial-sector writes, which bounded the
// kernel more than the decoding itself.
#include <cuda_fp16.h>

#include "cg_common.cuh"

namespace cg {
namespace {

constexpr int kUnitGroups = 32;
constexpr int kDeltaPerGroup = kGroup - 1;             // 9
constexpr int kWarps = 1 + kDeltaPerGroup;             // anchor warp + 9 delta warps
constexpr int kThreads = 32 * kWarps;                  // 320
constexpr int kUnitTokens = kUnitGroups * kGroup;      // 320
constexpr uint32_t kCumBuf = 800;                      // bytes per compacted-table buffer
constexpr uint32_t kRingBytes = 64;                    // per thread: 4 blocks of 16 bytes
constexpr uint32_t kRingBlocks = kRingBytes / 16;
constexpr uint32_t kRingWords = kRingBytes / 2;
constexpr uint32_t kRingStride = kRingBytes + 16;       // + a copy of slot 0 after slot 3

// Dynamic shared memory layout (byte offsets), a function of H and D.
struct DecSmem {
  uint32_t tbl;     // u32 [3][4096]  slot tables, packed (u << 24) | (f << 12) | (slot - cum)
  uint32_t ahat;    // f32 [2][32][D + 4]  reconstructed anchors of the last two heads
  uint32_t ring;    // u8  [320][80]  per-thread word rings: 4 slots + a mirror of slot 0
  uint32_t cum;     // [2] x {u16 pcum[257], u8 psym[256], i32 nz}: the next two heads' present
                    //        symbols in order and their cumulative frequencies
  uint32_t zs;      // f32 [2][2][D]  zero points and scales of the anchor warp's next heads
  uint32_t single;  // i32 [H]        symbol of a one-symbol table, else -1
  uint32_t total;
};

__host__ __device__ inline uint32_t al16(uint32_t v) { return (v + 15u) & ~15u; }

__host__ __device__ inline DecSmem dec_smem(int H, int D) {
  DecSmem s;
  s.tbl = 0;
  s.ahat = al16(s.tbl + 3u * 4096u * 4u);
  s.ring = al16(s.ahat + 2u * kUnitGroups * uint32_t(D + 4) * 4u);
  s.cum = al16(s.ring + uint32_t(kThreads) * kRingStride);
  s.zs = al16(s.cum + 2u * kCumBuf);
  s.single = al16(s.zs + 4u * uint32_t(D) * 4u);
  s.total = al16(s.single + uint32_t(H) * 4u);
  return s;
}

// ---- stream ring ------------------------------------------------------------
// Word q of the stream (absolute u16 index in the container) lives at ring byte
// offset 2 * (q mod 32): block b = q / 8 occupies slot b mod 4.
struct Ring {
  const uint8_t* gbase;  // container start (16-byte aligned)
  uint32_t rb;           // shared-memory address of this thread's ring (16-byte aligned)
  uint32_t fb;           // next 16-byte block of the container to request
  uint32_t lim;          // number of 16-byte blocks in the container
};

// Request the next block if the ring has room (predicated, no branch), then
// close the group.  A block landing in slot 0 is also copied to the mirror
// slot after slot 3, so that a step's reads run past the end of slot 3 without
// wrapping.
__device__ __forceinline__ void ring_issue(Ring& r, uint32_t p) {
  const uint32_t want = min((p >> 3) + kRingBlocks, r.lim);
  const uint32_t dst = r.rb + (r.fb & (kRingBlocks - 1)) * 16u;
  const uint8_t* src = r.gbase + uint64_t(r.fb) * 16u;
  asm volatile(
      "{\n\t"
      ".reg .pred p, m;\n\t"
      ".reg .u32 t;\n\t"
      "setp.lt.u32 p, %0, %1;\n\t"
      "and.b32 t, %0, 3;\n\t"
      "setp.eq.and.u32 m, t, 0, p;\n\t"
      "@p cp.async.cg.shared.global [%2], [%3], 16;\n\t"
      "@m cp.async.cg.shared.global [%4], [%3], 16;\n\t"
      "@p add.u32 %0, %0, 1;\n\t"
      "cp.async.commit_group;\n\t"
      "}\n"
      : "+r"(r.fb)
      : "r"(want), "r"(dst), "l"(src), "r"(r.rb + kRingBytes)
      : "memory");
}

__device__ __forceinline__ void ring_wait_two_steps() {
  asm volatile("cp.async.wait_group 2;\n" ::: "memory");
}

__device__ __forceinline__ void ring_wait_all() {
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u16 %0, [%1];\n" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ring_addr(const Ring& r, uint32_t q) {
  return r.rb + ((q & (kRingWords - 1)) << 1);
}

// Compacted table of one head: the present symbols in increasing order
// (psym), their cumulative frequencies (pcum, with pcum[nz] = 4096) and nz.
struct CumBuf {
  uint16_t* pcum;
  uint8_t* psym;
  int* nz;
};

__device__ __forceinline__ CumBuf cum_buf(uint8_t* base) {
  return CumBuf{reinterpret_cast<uint16_t*>(base), base + 520, reinterpret_cast<int*>(base + 784)};
}

// One warp turns a head's 256 frequencies (already in registers: lane holds
// symbols 8 lane .. 8 lane + 7) into its compacted table.
__device__ __forceinline__ void cum_compact(const uint4 raw, CumBuf cb, int lane) {
  const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t f[8];
  uint32_t local = 0, present = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = wv[i] & 0xFFFF;
    f[2 * i + 1] = wv[i] >> 16;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    local += f[i];
    present += f[i] != 0;
  }
  uint32_t incl = local, pincl = present;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    const uint32_t pv = __shfl_up_sync(0xFFFFFFFFu, pincl, o);
    if (lane >= o) {
      incl += v;
      pincl += pv;
    }
  }
  uint32_t run = incl - local, at = pincl - present;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (f[i] != 0) {
      cb.pcum[at] = uint16_t(run);
      cb.psym[at] = uint8_t(lane * 8 + i);
      ++at;
    }
    run += f[i];
  }
  if (lane == 31) {
    cb.pcum[pincl] = uint16_t(kM);
    *cb.nz = int(pincl);
  }
}

// Fill the 4096-entry slot table of one head: threads 0..255 each write 16
// consecutive slots with four 16-byte stores.  The symbol of the first slot is
// found by binary search over the present symbols' cumulative frequencies;
// each later slot advances at most one present symbol.
__device__ __forceinline__ void fill_table(uint32_t* tbl, CumBuf cb, int tid) {
  if (tid >= 256) return;
  const int s0 = tid * 16;
  int lo = 0, hi = *cb.nz;  // pcum[lo] <= s0 < pcum[hi]; pcum[nz] == 4096
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (int(cb.pcum[mid]) <= s0) lo = mid; else hi = mid;
  }
  int i = lo;
  int cc = cb.pcum[i], cn = cb.pcum[i + 1];
  uint32_t u = cb.psym[i];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t ent[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int s = s0 + 4 * q + k;
      if (cn <= s) {  // one step reaches the next present symbol
        ++i;
        cc = cn;
        cn = cb.pcum[i + 1];
        u = cb.psym[i];
      }
      ent[k] = (u << 24) | (uint32_t(cn - cc) << 12) | uint32_t(s - cc);
    }
    *reinterpret_cast<uint4*>(tbl + s0 + 4 * q) = make_uint4(ent[0], ent[1], ent[2], ent[3]);
  }
}

// One rANS decode step: returns the packed table entry of the decoded symbol.
// The refill is predicated, not branched: x = (x << 16) | w, advance the ring
// address ra and load the next word.  Within a step ra never wraps: it starts
// the step inside the 64-byte ring and a step reads at most 16 bytes, which
// may run into the mirror of slot 0.
__device__ __forceinline__ uint32_t rans_step(uint32_t& x, uint32_t& ra, uint32_t& w,
                                              const uint32_t* __restrict__ tbl) {
  const uint32_t e = tbl[x & (kM - 1)];
  x = ((e >> 12) & (kM - 1)) * (x >> kProbBits) + (e & (kM - 1));
  asm volatile(
      "{\n\t"
      ".reg .pred p;\n\t"
      "setp.lt.u32 p, %0, %3;\n\t"
      "@p prmt.b32 %0, %2, %0, 0x5410;\n\t"
      "@p add.u32 %1, %1, 2;\n\t"
      "@p ld.shared.u16 %2, [%1];\n\t"
      "}\n"
      : "+r"(x), "+r"(ra), "+r"(w)
      : "n"(kRansL));
  return e;
}

// Start of a step: bring the read address back into the 64-byte ring (the word
// under it is the same in slot 0 and in its mirror).
__device__ __forceinline__ uint32_t ring_rebase(uint32_t ra, uint32_t rb) {
  return rb + ((ra - rb) & (kRingBytes - 1));
}

// (float)(u - 127) for the symbol u in the entry's top byte: the bits
// 0x4B0000uu are the float 2^23 + u, and subtracting 2^23 + 127 is exact.
__device__ __forceinline__ float sym_value(uint32_t e) {
  return __fsub_rn(__uint_as_float(__byte_perm(e, 0x4B000000u, 0x7653)), 8388735.0f);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Stream position of a thread: p (absolute word index of the next unread
// word, kept per step) and ra (its ring address, advanced per refill).
struct Pos {
  uint32_t p, ra, w;
};

// 32-byte store of 16 fp16 values (one full sector); two 16-byte stores when
// the destination is only 16-byte aligned.
__device__ __forceinline__ void store16h(uint16_t* dst, const uint32_t (&hv)[8], bool al32) {
  if (al32) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"l"(dst),
                 "r"(hv[0]), "r"(hv[1]), "r"(hv[2]), "r"(hv[3]), "r"(hv[4]), "r"(hv[5]),
                 "r"(hv[6]), "r"(hv[7])
                 : "memory");
  } else {
    *reinterpret_cast<uint4*>(dst) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    *reinterpret_cast<uint4*>(dst + 8) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
  }
}

// The symbol u = q + 127 of a packed slot entry (format 2's first pass stores
// the symbols themselves, as u16, in the destination).
__device__ __forceinline__ uint32_t pack_codes(uint32_t e0, uint32_t e1) {
  return (e0 >> 24) | ((e1 >> 8) & 0x00FF0000u);
}

// Delta lane: decode head h of its stream in steps of 8 values; the values of
// two steps leave as one 32-byte store.  CODES: the symbols instead of values.
template <bool CODES>
__device__ __forceinline__ void decode_delta_head(uint32_t& x, Pos& ps, Ring& r,
                                                  const uint32_t* __restrict__ tbl, float step,
                                                  const float* __restrict__ arow,
                                                  uint16_t* __restrict__ orow, int D, bool al32) {
  for (int d0 = 0; d0 < D; d0 += 16) {
    uint32_t hv[8];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int dd = d0 + 8 * half;
      ring_issue(r, ps.p);
      ring_wait_two_steps();
      ps.ra = ring_rebase(ps.ra, r.rb);
      const uint32_t ra0 = ps.ra;
      const float4 a0 = *reinterpret_cast<const float4*>(arow + dd);
      const float4 a1 = *reinterpret_cast<const float4*>(arow + dd + 4);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
      for (int k = 0; k < 8; k += 2) {
        const uint32_t e0 = rans_step(x, ps.ra, ps.w, tbl);
        const uint32_t e1 = rans_step(x, ps.ra, ps.w, tbl);
        if constexpr (CODES) {
          hv[4 * half + (k >> 1)] = pack_codes(e0, e1);
        } else {
          const float v0 = __fadd_rn(a[k], __fmul_rn(sym_value(e0), step));
          const float v1 = __fadd_rn(a[k + 1], __fmul_rn(sym_value(e1), step));
          hv[4 * half + (k >> 1)] = pack_half2(v0, v1);
        }
      }
      ps.p += (ps.ra - ra0) >> 1;
    }
    store16h(orow + d0, hv, al32);
  }
}

// Anchor lane: decode head h, write fp16(a) and keep a (fp32) for the deltas.
// zp and sc point at the head's zero points and scales staged in shared memory.
// CODES: store the symbols only (format 2 rebuilds the values afterwards).
template <bool CODES>
__device__ __forceinline__ void decode_anchor_head(uint32_t& x, Pos& ps, Ring& r,
                                                   const uint32_t* __restrict__ tbl,
                                                   const float* __restrict__ zp,
                                                   const float* __restrict__ sc,
                                                   float* __restrict__ arow,
                                                   uint16_t* __restrict__ orow, int D, bool al32) {
  for (int d0 = 0; d0 < D; d0 += 16) {
    uint32_t hv[8];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int dd = d0 + 8 * half;
      ring_issue(r, ps.p);
      ring_wait_two_steps();
      ps.ra = ring_rebase(ps.ra, r.rb);
      const uint32_t ra0 = ps.ra;
      const float4 z0 = *reinterpret_cast<const float4*>(zp + dd);
      const float4 z1 = *reinterpret_cast<const float4*>(zp + dd + 4);
      const float4 s0 = *reinterpret_cast<const float4*>(sc + dd);
      const float4 s1 = *reinterpret_cast<const float4*>(sc + dd + 4);
      const float z[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
      const float s[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      if constexpr (CODES) {
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
          const uint32_t e0 = rans_step(x, ps.ra, ps.w, tbl);
          const uint32_t e1 = rans_step(x, ps.ra, ps.w, tbl);
          hv[4 * half + (k >> 1)] = pack_codes(e0, e1);
        }
        ps.p += (ps.ra - ra0) >> 1;
      } else {
        float v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t e = rans_step(x, ps.ra, ps.w, tbl);
          v[k] = __fadd_rn(z[k], __fmul_rn(sym_value(e), s[k]));
        }
        ps.p += (ps.ra - ra0) >> 1;
        *reinterpret_cast<float4*>(arow + dd) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4*>(arow + dd + 4) = make_float4(v[4], v[5], v[6], v[7]);
#pragma unroll
        for (int k = 0; k < 4; ++k) hv[4 * half + k] = pack_half2(v[2 * k], v[2 * k + 1]);
      }
    }
    store16h(orow + d0, hv, al32);
  }
}

// Header validation of one container (both decode kernels run it; every CTA
// of a chunk checks the same 64 bytes).  Returns 0 or the status to report.
__device__ int check_header(const uint8_t* base, const DecParams& p, cg_header& h) {
  const uint4* hp = reinterpret_cast<const uint4*>(base);
  uint4* hd = reinterpret_cast<uint4*>(&h);
  for (int i = 0; i < 4; ++i) hd[i] = __ldg(hp + i);
  const int L = p.L, H = p.H, D = p.D;
  const uint32_t want = p.adjacent ? CG_FORMAT_VERSION_ADJACENT : CG_FORMAT_VERSION;
  int err = 0;
  if (h.magic != CG_MAGIC || h.group != kGroup || h.prob_bits != kProbBits || h.reserved != 0 ||
      (h.version != CG_FORMAT_VERSION && h.version != CG_FORMAT_VERSION_ADJACENT))
    err = CG_ERR_CORRUPT;
  else if (h.version != want || h.level != uint32_t(p.level) ||
           h.num_layers != uint32_t(L) || h.num_kv_heads != uint32_t(H) ||
           h.head_dim != uint32_t(D) || h.chunk_tokens != uint32_t(p.C))
    err = CG_ERR_MISMATCH;  // the other format, or another level or shape
  else if (h.n_tokens < 1 || h.n_tokens > uint32_t(p.C))
    err = CG_ERR_CORRUPT;
  if (!err) {
    const Sections sec = sections(L, H, D, h.n_tokens);
    if (h.payload_bytes > 0xFFFFFFFFull || h.total_bytes > p.in_stride ||
        sec.payload + h.payload_bytes > h.total_bytes ||
        up16(sec.payload + h.payload_bytes) != h.total_bytes)
      err = CG_ERR_CORRUPT;
    else if (p.into && (h.token_start > uint64_t(p.total_tokens) ||
                        h.token_start + h.n_tokens > uint64_t(p.total_tokens)))
      err = CG_ERR_MISMATCH;
  }
  return err;
}

// Destination row (H*D values) of local token t of a chunk, or null when a
// paged destination's block table does not map it.
__device__ __forceinline__ uint16_t* dest_row(const DecParams& p, int chunk, int slab, int n,
                                              long long tstart, int t) {
  const int H = p.H, D = p.D;
  if (p.into == 1)
    return p.out + ((uint64_t(slab) * p.total_tokens + uint64_t(tstart) + t) * H) * D;
  if (p.into == 2) {
    const int64_t g = tstart + t;  // logical token g: row g mod P of page block_table[g / P]
    const int32_t page = __ldg(p.block_table + g / p.page_tokens);
    if (page < 0 || page >= p.num_pages) return nullptr;
    return p.out + (((uint64_t(slab) * p.num_pages + uint64_t(page)) * p.page_tokens +
                     uint64_t(g % p.page_tokens)) * H) * D;
  }
  return p.out + uint64_t(chunk) * (uint64_t(p.L) * 2 * p.C * H * D) +
         ((uint64_t(slab) * n + t) * H) * D;
}

template <bool CODES>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const DecParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int s_ok, s_n, s_bad;
  __shared__ long long s_tstart;
  __shared__ unsigned long long s_total;

  const int tid = threadIdx.x;
  const int unit = blockIdx.x % p.units_per_slab;
  int rest = blockIdx.x / p.units_per_slab;
  const int kv = rest & 1;
  rest >>= 1;
  const int l = rest % p.L;
  const int chunk = rest / p.L;
  const int L = p.L, H = p.H, D = p.D;
  const uint8_t* base = p.in + uint64_t(chunk) * p.in_stride;

  if (tid == 0) {
    cg_header h;
    const int err = check_header(base, p, h);
    if (err) set_status(p.status, err);
    s_ok = !err;
    s_n = int(h.n_tokens);
    s_tstart = (long long)h.token_start;
    s_total = h.total_bytes;
    s_bad = 0;
  }
  __syncthreads();
  if (!s_ok) return;
  const int n = s_n;
  const int unit_t0 = unit * kUnitTokens;
  if (unit_t0 >= n) return;

  const Sections sec = sections(L, H, D, n);
  const DecSmem sm = dec_smem(H, D);
  uint32_t* tbl = reinterpret_cast<uint32_t*>(smem + sm.tbl);
  float* ahat = reinterpret_cast<float*>(smem + sm.ahat);
  int* single = reinterpret_cast<int*>(smem + sm.single);
  const int astride = D + 4;
  const int warp = tid >> 5, lane = tid & 31;
  const int slab = l * 2 + kv;

  // Validate every frequency table of this (l, kv) and note one-symbol tables.
  const uint16_t* freq = reinterpret_cast<const uint16_t*>(base + sec.freq) + size_t(slab) * H * 256;
  for (int h = warp; h < H; h += kWarps) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(freq + h * 256) + lane);
    const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t local = 0;
    int one = -1;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t f = (wv[i >> 1] >> (16 * (i & 1))) & 0xFFFF;
      local += f;
      if (f == kM) one = lane * 8 + i;
      if (f > kM) bad = true;
    }
    if (lane == 31 && (wv[3] >> 16) != 0) bad = true;  // symbol 255 never exists
    const uint32_t total = __reduce_add_sync(0xFFFFFFFFu, local);
    one = __reduce_max_sync(0xFFFFFFFFu, one);
    if (lane == 0) single[h] = one;
    if (__any_sync(0xFFFFFFFFu, bad) || total != kM) {
      if (lane == 0) s_bad = 1;
    }
  }
  const float step = step_of(p.level, l, L);
  // 32-byte stores need a 32-byte aligned destination (rows are multiples of 32 bytes)
  const bool al32 = (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0;
  __syncthreads();
  if (s_bad) {
    if (tid == 0) set_status(p.status, CG_ERR_CORRUPT);
    return;
  }
  uint8_t* cumb = smem + sm.cum;
  if (warp < 2 && warp < H)
    cum_compact(__ldg(reinterpret_cast<const uint4*>(freq + warp * 256) + lane),
                cum_buf(cumb + warp * kCumBuf), lane);
  __syncthreads();
  fill_table(tbl, cum_buf(cumb), tid);

  // This thread's stream.
  int g_local, token;
  if (warp == 0) {
    g_local = lane;
    token = unit_t0 + kGroup * lane;
  } else {
    const int k = (warp - 1) * 32 + lane;
    g_local = k / kDeltaPerGroup;
    token = unit_t0 + kGroup * g_local + 1 + k % kDeltaPerGroup;
  }
  bool active = token < n;
  const uint32_t* offs = reinterpret_cast<const uint32_t*>(base + sec.offsets);
  // Destination row of this thread's token (a paged pool's block table may
  // leave it unmapped: nothing is written for it).
  uint16_t* orow = p.out;
  if (active) {
    orow = dest_row(p, chunk, slab, n, s_tstart, token);
    if (orow == nullptr) {
      set_status(p.status, CG_ERR_MISMATCH);
      active = false;
      orow = p.out;
    }
  }
  Ring ring;
  ring.gbase = base;
  const uint32_t rings = uint32_t(__cvta_generic_to_shared(smem + sm.ring));
  ring.rb = rings + uint32_t(tid) * kRingStride;
  ring.lim = uint32_t(s_total / 16);
  ring.fb = 0;
  Pos ps{0u, ring.rb, 0u};
  uint32_t pend = 0, x = kRansL;
  if (active) {
    const uint64_t s = uint64_t(slab) * n + token;
    const uint32_t o0 = __ldg(offs + s), o1 = __ldg(offs + s + 1);
    const uint64_t payload = s_total - sec.payload;  // includes the final padding
    if (o1 < o0 || uint64_t(o1) > payload || ((o1 - o0) & 1u) || o1 - o0 < 4) {
      set_status(p.status, CG_ERR_CORRUPT);
      active = false;
    } else {
      uint32_t pw = uint32_t((sec.payload + o0) / 2);
      pend = uint32_t((sec.payload + o1) / 2);
      ring.fb = pw >> 3;
      for (uint32_t i = 0; i < kRingBlocks; ++i) ring_issue(ring, pw);
      ring_wait_all();
      x = (lds_u16(ring_addr(ring, pw)) << 16) | lds_u16(ring_addr(ring, pw + 1));
      pw += 2;
      ps.p = pw;
      ps.ra = ring_addr(ring, pw);
      ps.w = lds_u16(ps.ra);
      if (x < kRansL) {
        set_status(p.status, CG_ERR_CORRUPT);
        active = false;
      }
    }
  }
  const float* zp_sec = reinterpret_cast<const float*>(base + sec.zp) + size_t(slab) * H * D;
  const float* sc_sec = reinterpret_cast<const float*>(base + sec.scale) + size_t(slab) * H * D;
  float* zs = reinterpret_cast<float*>(smem + sm.zs);  // [2][{zp, scale}][D]
  for (int i = tid; i < 2 * D; i += kThreads)
    zs[i] = i < D ? __ldg(zp_sec + i) : __ldg(sc_sec + (i - D));
  __syncthreads();

  for (int it = 0; it <= H; ++it) {
    // Global loads for the next heads are issued first and consumed after this
    // iteration's decode, so their latency never delays the barrier.
    const bool scan_warp = it + 2 < H && warp == it % kWarps;
    uint4 fq = make_uint4(0, 0, 0, 0);
    if (scan_warp) fq = __ldg(reinterpret_cast<const uint4*>(freq + (it + 2) * 256) + lane);
    float zv[2] = {0.0f, 0.0f};
    const bool stage = it + 1 < H;
    if (stage) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int i = tid + j * kThreads;
        if (i < 2 * D)
          zv[j] = i < D ? __ldg(zp_sec + (it + 1) * D + i) : __ldg(sc_sec + (it + 1) * D + (i - D));
      }
      fill_table(tbl + ((it + 1) % 3) * kM, cum_buf(cumb + ((it + 1) & 1) * kCumBuf), tid);
    }
    if (warp == 0) {
      if (it < H && active) {
        const int h = it;
        const uint32_t* tb = tbl + (h % 3) * kM;
        float* arow = ahat + ((h & 1) * kUnitGroups + g_local) * astride;
        const float* zh = zs + (h & 1) * 2 * D;
        const int one = single[h];
        if (one >= 0 && CODES) {
          const uint32_t cc = uint32_t(one) * 0x10001u;
          for (int d0 = 0; d0 < D; d0 += 8)
            *reinterpret_cast<uint4*>(orow + h * D + d0) = make_uint4(cc, cc, cc, cc);
        } else if (one >= 0) {
          const float c = float(one - 127);
          for (int d0 = 0; d0 < D; d0 += 8) {
            float v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = __fadd_rn(zh[d0 + k], __fmul_rn(c, zh[D + d0 + k]));
#pragma unroll
            for (int k = 0; k < 8; ++k) arow[d0 + k] = v[k];
            *reinterpret_cast<uint4*>(orow + h * D + d0) =
                make_uint4(pack_half2(v[0], v[1]), pack_half2(v[2], v[3]),
                           pack_half2(v[4], v[5]), pack_half2(v[6], v[7]));
          }
        } else {
          decode_anchor_head<CODES>(x, ps, ring, tb, zh, zh + D, arow, orow + h * D, D, al32);
        }
      }
    } else if (it >= 1 && active) {
      const int h = it - 1;
      const uint32_t* tb = tbl + (h % 3) * kM;
      const float* arow = ahat + ((h & 1) * kUnitGroups + g_local) * astride;
      const int one = single[h];
      if (one >= 0 && CODES) {
        const uint32_t cc = uint32_t(one) * 0x10001u;
        for (int d0 = 0; d0 < D; d0 += 8)
          *reinterpret_cast<uint4*>(orow + h * D + d0) = make_uint4(cc, cc, cc, cc);
      } else if (one >= 0) {
        const float v = __fmul_rn(float(one - 127), step);
        for (int d0 = 0; d0 < D; d0 += 8) {
          uint32_t hv[4];
#pragma unroll
          for (int k = 0; k < 8; k += 2)
            hv[k >> 1] = pack_half2(__fadd_rn(arow[d0 + k], v), __fadd_rn(arow[d0 + k + 1], v));
          *reinterpret_cast<uint4*>(orow + h * D + d0) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        }
      } else {
        decode_delta_head<CODES>(x, ps, ring, tb, step, arow, orow + h * D, D, al32);
      }
    }
    if (scan_warp) cum_compact(fq, cum_buf(cumb + (it & 1) * kCumBuf), lane);
    if (stage) {
      float* zn = zs + ((it + 1) & 1) * 2 * D;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int i = tid + j * kThreads;
        if (i < 2 * D) zn[i] = zv[j];
      }
    }
    __syncthreads();
  }
  ring_wait_all();
  if (active && (x != kRansL || ps.p != pend)) set_status(p.status, CG_ERR_CORRUPT);
}

// ---- format 2, second pass -------------------------------------------------
// decode_kernel<true> has left every value's symbol u = q + 127 (a u16) in its
// destination slot.  One thread per (anchor group, 8 channels of the token
// row) rebuilds the group's chain in place: the anchor a = zp + c * scale,
// then x^_t = x^_(t-1) + q_t * step for the group's later tokens, each sum and
// product rounded to nearest (no contraction), each value stored as fp16.  The
// ten rows' symbols are loaded before the first store, so a thread keeps ten
// 16-byte loads in flight; a warp covers 512 contiguous bytes of each row.
constexpr int kChainThreads = 256;

__global__ void __launch_bounds__(kChainThreads) chain_kernel(const DecParams p,
                                                              const int blocks_per_slab) {
  __shared__ int s_ok, s_n;
  __shared__ long long s_tstart;
  const int tid = threadIdx.x;
  const int part = blockIdx.x % blocks_per_slab;
  const int rest = blockIdx.x / blocks_per_slab;
  const int slab = rest % (2 * p.L);
  const int chunk = rest / (2 * p.L);
  const int L = p.L, H = p.H, D = p.D;
  const uint8_t* base = p.in + uint64_t(chunk) * p.in_stride;
  if (tid == 0) {
    cg_header h;
    s_ok = check_header(base, p, h) == 0;  // the decode pass has reported any error
    s_n = int(h.n_tokens);
    s_tstart = (long long)h.token_start;
  }
  __syncthreads();
  if (!s_ok) return;
  const int n = s_n;
  const int rb = H * D / 8;  // 8-channel blocks of a token row
  const int64_t w = int64_t(part) * kChainThreads + tid;
  if (w >= int64_t((n + kGroup - 1) / kGroup) * rb) return;
  const int g = int(w / rb), c0 = int(w % rb) * 8;
  const int t0 = g * kGroup, ntok = min(kGroup, n - t0);
  const Sections sec = sections(L, H, D, n);
  const float* zp = reinterpret_cast<const float*>(base + sec.zp) + uint64_t(slab) * H * D + c0;
  const float* sc = reinterpret_cast<const float*>(base + sec.scale) + uint64_t(slab) * H * D + c0;
  const float4 z0 = __ldg(reinterpret_cast<const float4*>(zp));
  const float4 z1 = __ldg(reinterpret_cast<const float4*>(zp + 4));
  const float4 s0 = __ldg(reinterpret_cast<const float4*>(sc));
  const float4 s1 = __ldg(reinterpret_cast<const float4*>(sc + 4));
  const float z[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
  const float sa[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  const float step = step_of(p.level, slab >> 1, L);

  uint16_t* rows[kGroup];
  uint4 cv[kGroup];
#pragma unroll
  for (int r = 0; r < kGroup; ++r) {
    rows[r] = r < ntok ? dest_row(p, chunk, slab, n, s_tstart, t0 + r) : nullptr;
    cv[r] = rows[r] ? *reinterpret_cast<const uint4*>(rows[r] + c0) : make_uint4(0, 0, 0, 0);
  }
  float x[8];
#pragma unroll
  for (int r = 0; r < kGroup; ++r) {
    if (rows[r] == nullptr) break;  // end of the chunk (or an unmapped page)
    const uint32_t cw[4] = {cv[r].x, cv[r].y, cv[r].z, cv[r].w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float q = float(int((cw[k >> 1] >> (16 * (k & 1))) & 0xFFFFu) - 127);
      x[k] = r == 0 ? __fadd_rn(z[k], __fmul_rn(q, sa[k])) : __fadd_rn(x[k], __fmul_rn(q, step));
    }
    *reinterpret_cast<uint4*>(rows[r] + c0) =
        make_uint4(pack_half2(x[0], x[1]), pack_half2(x[2], x[3]), pack_half2(x[4], x[5]),
                   pack_half2(x[6], x[7]));
  }
}

}  // namespace

cudaError_t launch_decode(const DecParams& p, cudaStream_t stream) {
  const DecSmem sm = dec_smem(p.H, p.D);
  auto* kern = p.adjacent ? decode_kernel<true> : decode_kernel<false>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm.total));
  if (err != cudaSuccess) return err;
  const uint64_t blocks = uint64_t(p.num_chunks) * p.L * 2 * p.units_per_slab;
  kern<<<unsigned(blocks), kThreads, sm.total, stream>>>(p);
  if ((err = cudaGetLastError()) != cudaSuccess || !p.adjacent) return err;
  const uint64_t work = uint64_t((p.C + kGroup - 1) / kGroup) * (p.H * p.D / 8);
  const int per_slab = int((work + kChainThreads - 1) / kChainThreads);
  chain_kernel<<<unsigned(uint64_t(p.num_chunks) * p.L * 2 * per_slab), kChainThreads, 0,
                 stream>>>(p, per_slab);
  return cudaGetLastError();
}

int decode_units_per_slab(int C) {
  const int groups = (C + kGroup - 1) / kGroup;
  return (groups + kUnitGroups - 1) / kUnitGroups;
}

}  // namespace cg
