// decode.cu -- fused rANS decode -> dequantise -> fp16 store: cg_decode,
// cg_decode_into, cg_decode_into_paged, and the format-2 calls
// cg_decode_adjacent / cg_decode_adjacent_into.
//
// [Practice] 2.3 (parallel decode): the receiver decodes on the GPU with one
// thread per token and hands the result to the thread that fills the model's
// KV cache.  Here one thread owns one rANS stream, i.e. one (layer, K/V,
// token), and the same kernel writes the fp16 values into the destination
// layout, so decode and fill are one kernel.
//
// CTA = one "unit": 32 anchor groups (320 tokens) of one (chunk, layer, K/V);
// thread t decodes the stream of local token t (anchors and deltas alike).
// Every stream holds H*D symbols in [h][d] order and every head has its own
// frequency table, so the CTA walks the heads in lockstep.  Each head is
// taken in two slices of D/2 channels, two phases per slice:
//
//   phase A  every thread decodes the slice's D/2 symbols of its stream and
//            leaves the byte codes u = q + 127 in shared memory, codes[t][d];
//            the only shared-memory traffic is the slot-table lookup, the word
//            refill and one 8-byte code store per 8 symbols.
//   phase B  the threads turn the slice's codes into fp16.  A work item is
//            (anchor group g, 8 channels): the anchor's values
//            a = zp + (float)c * scale, then the nine deltas a + (float)q * step
//            (format 2: each delta against the previous token's value), all
//            fp32 with IEEE round-to-nearest adds and multiplies (no
//            contraction), each row's 8 values leaving as one 16-byte store;
//            consecutive lanes take consecutive channel blocks, so a warp's
//            stores cover whole row segments.  After the head's last slice the
//            slot table is rebuilt for head h + 1 (phase A of head h no longer
//            reads it) and the zero points / scales of head h + 1 are staged.
//
// A __syncthreads separates the phases (four per head).  Anchors get no
// special treatment in phase A, and the reconstructed anchors never leave the
// registers of the phase-B item, so the work of a head is spread evenly over
// the CTA.  Half a head of codes keeps a CTA at about 72 KB of shared memory,
// so three CTAs (30 warps) share an SM.
//
// Compressed words reach a thread through a 64-byte ring in shared memory
// (four 16-byte blocks, plus a copy of the first block after the last, so that
// the reads of one step never wrap).  Every 8 symbols the thread issues at most one
// cp.async for the next block of its stream and waits only for the blocks
// issued two steps earlier; since 8 symbols consume at most 8 words (one
// block), the words a step can read were always requested at least two steps
// before, so global-memory latency stays off the decode chain.
#include <cuda_fp16.h>

#include "cg_common.cuh"

namespace cg {
namespace {

constexpr int kUnitGroups = 32;
constexpr int kThreads = kUnitGroups * kGroup;         // 320: one stream per thread
constexpr int kWarps = kThreads / 32;                  // 10
constexpr int kUnitTokens = kThreads;
constexpr uint32_t kCumBuf = 800;                      // bytes per compacted-table buffer
constexpr uint32_t kRingBytes = 64;                    // per thread: 4 blocks of 16 bytes
constexpr uint32_t kRingBlocks = kRingBytes / 16;
constexpr uint32_t kRingWords = kRingBytes / 2;
constexpr uint32_t kRingStride = kRingBytes + 16;       // + a copy of slot 0 after slot 3

// Dynamic shared memory layout (byte offsets), a function of H and D.
struct DecSmem {
  uint32_t tbl;     // u32 [4096]     slot table of the current head, packed
                    //                (u << 24) | (f << 12) | (slot - cum)
  uint32_t codes;   // u8  [320][D + 8]  symbols u of the current head, one row per token
  uint32_t ring;    // u8  [320][80]  per-thread word rings: 4 slots + a mirror of slot 0
  uint32_t cum;     // [2] x {u16 pcum[257], u8 psym[256], i32 nz}: compacted tables of
                    //        the next heads (present symbols in order, cumulative freqs)
  uint32_t zs;      // f32 [2][2][D]  zero points and scales of the current and next head
  uint32_t rows;    // u64 [320]      destination row of each token (0: not written)
  uint32_t ok;      // u8  [320]      1 when the token's stream is being decoded
  uint32_t gok;     // u8  [32]       1 when every stream of the anchor group is
  uint32_t single;  // i32 [H]        symbol of a one-symbol table, else -1
  uint32_t total;
};

__host__ __device__ inline uint32_t al16(uint32_t v) { return (v + 15u) & ~15u; }

// A head is decoded in kSlices slices of D / kSlices channels (two phases
// each), so the code buffer holds one slice: that keeps a CTA's shared memory
// small enough for three CTAs per SM.
constexpr int kSlices = 2;

__host__ __device__ inline uint32_t codes_stride(int D) { return uint32_t(D / kSlices) + 8u; }

__host__ __device__ inline DecSmem dec_smem(int H, int D) {
  DecSmem s;
  s.tbl = 0;
  s.codes = s.tbl + 4096u * 4u;
  s.ring = al16(s.codes + uint32_t(kThreads) * codes_stride(D));
  s.cum = al16(s.ring + uint32_t(kThreads) * kRingStride);
  s.zs = al16(s.cum + 2u * kCumBuf);
  s.rows = al16(s.zs + 4u * uint32_t(D) * 4u);
  s.ok = al16(s.rows + uint32_t(kThreads) * 8u);
  s.gok = al16(s.ok + uint32_t(kThreads));
  s.single = al16(s.gok + uint32_t(kUnitGroups));
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
                                              uint32_t tbl_s) {
  uint32_t e;
  asm volatile("ld.shared.u32 %0, [%1];\n"
               : "=r"(e)
               : "r"(tbl_s + ((x & (kM - 1)) << 2))
               : "memory");
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

// The symbols u (top bytes of four slot entries) as four bytes of one word.
__device__ __forceinline__ uint32_t pack4(uint32_t e0, uint32_t e1, uint32_t e2, uint32_t e3) {
  return __byte_perm(__byte_perm(e0, e1, 0x0073), __byte_perm(e2, e3, 0x0073), 0x5410);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Header validation of one container (every CTA of a chunk checks the same
// 64 bytes).  Returns 0 or the status to report.
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

// Phase A for one head: decode D symbols of the thread's stream with the slot
// table tb and leave their codes in the thread's row of the code buffer.
__device__ __forceinline__ void decode_codes(uint32_t& x, uint32_t& p, uint32_t& ra,
                                             uint32_t& w, Ring& r, uint32_t tb_s,
                                             uint32_t crow_s, int D) {
  for (int d0 = 0; d0 < D; d0 += 8) {
    ring_issue(r, p);
    ring_wait_two_steps();
    ra = ring_rebase(ra, r.rb);
    const uint32_t ra0 = ra;
    const uint32_t e0 = rans_step(x, ra, w, tb_s);
    const uint32_t e1 = rans_step(x, ra, w, tb_s);
    const uint32_t e2 = rans_step(x, ra, w, tb_s);
    const uint32_t e3 = rans_step(x, ra, w, tb_s);
    const uint32_t e4 = rans_step(x, ra, w, tb_s);
    const uint32_t e5 = rans_step(x, ra, w, tb_s);
    const uint32_t e6 = rans_step(x, ra, w, tb_s);
    const uint32_t e7 = rans_step(x, ra, w, tb_s);
    p += (ra - ra0) >> 1;
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};\n" ::"r"(crow_s + uint32_t(d0)),
                 "r"(pack4(e0, e1, e2, e3)), "r"(pack4(e4, e5, e6, e7))
                 : "memory");
  }
}

// Packed fp32 pair arithmetic (sm_100 f32x2): each component rounds like the
// scalar instruction with the same modifier.  A packed multiply feeding a
// packed add did not give RN(a + RN(q * s)) on sm_100a (most cancelling sums
// differed, as from a fused multiply-add), even with the rounding modifier
// written out, so a product is only ever added with the scalar __fadd_rn,
// which is never contracted.
__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// (float)(u - 127) for bytes K and K + 1 of a word of codes: the bits
// 0x4B0000uu are the float 2^23 + u, and subtracting 2^23 + 127 is exact.
template <int K>
__device__ __forceinline__ float2 code_pair(uint32_t w) {
  const float2 biased = make_float2(__uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u | K)),
                                    __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u | (K + 1))));
  return add2_rn(biased, make_float2(-8388735.0f, -8388735.0f));
}

// Eight values a[k] + (float)q[k] * s[k] of the eight codes in c, as fp16 (four
// words): codes and products two channels per packed instruction, the final
// adds one channel at a time.
template <bool SCALAR_S>
__device__ __forceinline__ uint4 dequant8(const uint2 c, const float2 (&a)[4], const float2* s,
                                          float2 (&v)[4]) {
  const uint32_t cw[2] = {c.x, c.y};
  uint32_t h[4];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float2 q0 = code_pair<0>(cw[i]);
    const float2 q1 = code_pair<2>(cw[i]);
    const float2 p0 = mul2_rn(q0, SCALAR_S ? s[0] : s[2 * i + 0]);
    const float2 p1 = mul2_rn(q1, SCALAR_S ? s[0] : s[2 * i + 1]);
    v[2 * i + 0] = make_float2(__fadd_rn(a[2 * i + 0].x, p0.x), __fadd_rn(a[2 * i + 0].y, p0.y));
    v[2 * i + 1] = make_float2(__fadd_rn(a[2 * i + 1].x, p1.x), __fadd_rn(a[2 * i + 1].y, p1.y));
    h[2 * i + 0] = pack_half2(v[2 * i + 0].x, v[2 * i + 0].y);
    h[2 * i + 1] = pack_half2(v[2 * i + 1].x, v[2 * i + 1].y);
  }
  return make_uint4(h[0], h[1], h[2], h[3]);
}

// Where phase B writes: a flat destination (token t's row at row0 + t * HD)
// or, for a paged pool, the per-token rows in shared memory (0: unmapped).
struct RowMap {
  uint16_t* row0;
  uint64_t HD;
  const uint64_t* rows;
};

template <bool PAGED>
__device__ __forceinline__ uint16_t* row_of(const RowMap& m, int t) {
  if (PAGED) return reinterpret_cast<uint16_t*>(m.rows[t]);
  return m.row0 + uint64_t(t) * m.HD;
}

// Phase B for one head: fp16 values from the codes.  Item (group g, block b
// of 8 channels): the anchor's 8 values a = zp + (float)c * scale, then the
// same 8 channels of each later token of the group, a + (float)q * step
// (format 2: each against the previous token's values), each row leaving as
// one 16-byte store.  Consecutive lanes take consecutive blocks, so a warp's
// stores cover whole row segments.
// gok[g]: every stream of group g decodes; otherwise rows whose stream was
// rejected are skipped (format 2: the rest of the chain too), and a group whose
// anchor was rejected stays untouched.
template <bool ADJ, bool PAGED>
__device__ __forceinline__ void dequant_head(const uint8_t* __restrict__ codes, uint32_t cstride,
                                             const float* __restrict__ zh, const RowMap& rm,
                                             const uint8_t* __restrict__ ok,
                                             const uint8_t* __restrict__ gok, int ngroups,
                                             int ntok, int h, int D, int cbase, int DS,
                                             float step, int tid, int dq, int dr) {
  const int B8 = DS >> 3;
  int g = tid / B8, b = tid - g * B8;  // item tid, then steps of kThreads = dq * B8 + dr items
  for (; g < ngroups; g += dq, b += dr) {
    if (b >= B8) {
      b -= B8;
      if (++g >= ngroups) break;
    }
    const int t0 = g * kGroup;
    if (!ok[t0]) continue;
    const int c0 = 8 * b;      // column in the slice's code rows
    const int cz = cbase + c0;  // channel in the head
    float2 a[4], v[4];
    {
      const float4 z0 = *reinterpret_cast<const float4*>(zh + cz);
      const float4 z1 = *reinterpret_cast<const float4*>(zh + cz + 4);
      const float4 s0 = *reinterpret_cast<const float4*>(zh + D + cz);
      const float4 s1 = *reinterpret_cast<const float4*>(zh + D + cz + 4);
      const float2 z[4] = {make_float2(z0.x, z0.y), make_float2(z0.z, z0.w),
                           make_float2(z1.x, z1.y), make_float2(z1.z, z1.w)};
      const float2 sc[4] = {make_float2(s0.x, s0.y), make_float2(s0.z, s0.w),
                            make_float2(s1.x, s1.y), make_float2(s1.z, s1.w)};
      const uint2 c = *reinterpret_cast<const uint2*>(codes + t0 * cstride + c0);
      const uint4 hv = dequant8<false>(c, z, sc, a);
      uint16_t* r = row_of<PAGED>(rm, t0);
      if (!PAGED || r) *reinterpret_cast<uint4*>(r + h * D + cz) = hv;
    }
    const float2 st[1] = {make_float2(step, step)};
    const int tend = min(kGroup, ntok - t0);
    const uint8_t* cr = codes + t0 * cstride + c0;
    if (gok[g]) {
      // flat destinations: the rows of consecutive tokens are HD values apart
      uint16_t* fr = PAGED ? nullptr : row_of<false>(rm, t0) + (h * D + cz);
#pragma unroll
      for (int r = 1; r < kGroup; ++r) {
        if (r >= tend) break;
        const uint2 q = *reinterpret_cast<const uint2*>(cr + r * cstride);
        const uint4 hv = dequant8<true>(q, a, st, v);
        if (PAGED) {
          uint16_t* row = row_of<true>(rm, t0 + r);
          if (row) *reinterpret_cast<uint4*>(row + h * D + cz) = hv;
        } else {
          fr += rm.HD;
          *reinterpret_cast<uint4*>(fr) = hv;
        }
        if (ADJ) {
#pragma unroll
          for (int k = 0; k < 4; ++k) a[k] = v[k];
        }
      }
    } else {
      for (int r = 1; r < tend; ++r) {
        if (!ok[t0 + r]) {
          if (ADJ) break;  // the chain has lost a link: the rest of the group stays untouched
          continue;
        }
        const uint2 q = *reinterpret_cast<const uint2*>(cr + r * cstride);
        const uint4 hv = dequant8<true>(q, a, st, v);
        uint16_t* row = row_of<PAGED>(rm, t0 + r);
        if (!PAGED || row) *reinterpret_cast<uint4*>(row + h * D + cz) = hv;
        if (ADJ) {
#pragma unroll
          for (int k = 0; k < 4; ++k) a[k] = v[k];
        }
      }
    }
  }
}

template <bool ADJ, bool PAGED>
__global__ void __launch_bounds__(kThreads, 3) decode_kernel(const DecParams p) {
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
  const int ntok = min(kUnitTokens, n - unit_t0);   // tokens of this unit
  const int ngroups = (ntok + kGroup - 1) / kGroup;

  const Sections sec = sections(L, H, D, n);
  const DecSmem sm = dec_smem(H, D);
  uint32_t* tbl = reinterpret_cast<uint32_t*>(smem + sm.tbl);
  uint8_t* codes = smem + sm.codes;
  const uint32_t cstride = codes_stride(D);
  uint64_t* rows = reinterpret_cast<uint64_t*>(smem + sm.rows);
  uint8_t* okf = smem + sm.ok;
  uint8_t* gok = smem + sm.gok;
  int* single = reinterpret_cast<int*>(smem + sm.single);
  float* zs = reinterpret_cast<float*>(smem + sm.zs);  // [2][{zp, scale}][D]
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
  __syncthreads();
  if (s_bad) {
    if (tid == 0) set_status(p.status, CG_ERR_CORRUPT);
    return;
  }
  uint8_t* cumb = smem + sm.cum;
  if (warp < 2 && warp < H)
    cum_compact(__ldg(reinterpret_cast<const uint4*>(freq + warp * 256) + lane),
                cum_buf(cumb + warp * kCumBuf), lane);
  const float* zp_sec = reinterpret_cast<const float*>(base + sec.zp) + size_t(slab) * H * D;
  const float* sc_sec = reinterpret_cast<const float*>(base + sec.scale) + size_t(slab) * H * D;
  for (int i = tid; i < 2 * D; i += kThreads)
    zs[i] = i < D ? __ldg(zp_sec + i) : __ldg(sc_sec + (i - D));
  __syncthreads();
  fill_table(tbl, cum_buf(cumb), tid);

  // This thread's stream: local token unit_t0 + tid.
  const int token = unit_t0 + tid;
  bool active = tid < ntok;
  uint64_t orow = 0;
  if (active) {
    uint16_t* r = dest_row(p, chunk, slab, n, s_tstart, token);
    if (r == nullptr) set_status(p.status, CG_ERR_MISMATCH);  // unmapped page: not written
    orow = reinterpret_cast<uint64_t>(r);
  }
  const uint32_t* offs = reinterpret_cast<const uint32_t*>(base + sec.offsets);
  Ring ring;
  ring.gbase = base;
  const uint32_t rings = uint32_t(__cvta_generic_to_shared(smem + sm.ring));
  ring.rb = rings + uint32_t(tid) * kRingStride;
  ring.lim = uint32_t(s_total / 16);
  ring.fb = 0;
  uint32_t x = kRansL, pw = 0, pend = 0, ra = ring.rb, w = 0;
  if (active) {
    const uint64_t s = uint64_t(slab) * n + token;
    const uint32_t o0 = __ldg(offs + s), o1 = __ldg(offs + s + 1);
    const uint64_t payload = s_total - sec.payload;  // includes the final padding
    if (o1 < o0 || uint64_t(o1) > payload || ((o1 - o0) & 1u) || o1 - o0 < 4) {
      set_status(p.status, CG_ERR_CORRUPT);
      active = false;
    } else {
      pw = uint32_t((sec.payload + o0) / 2);
      pend = uint32_t((sec.payload + o1) / 2);
      ring.fb = pw >> 3;
      for (uint32_t i = 0; i < kRingBlocks; ++i) ring_issue(ring, pw);
      ring_wait_all();
      x = (lds_u16(ring_addr(ring, pw)) << 16) | lds_u16(ring_addr(ring, pw + 1));
      pw += 2;
      ra = ring_addr(ring, pw);
      w = lds_u16(ra);
      if (x < kRansL) {
        set_status(p.status, CG_ERR_CORRUPT);
        active = false;
      }
    }
  }
  if (PAGED) rows[tid] = orow;
  okf[tid] = active ? 1 : 0;
  const uint32_t tbl_s = uint32_t(__cvta_generic_to_shared(tbl));
  const uint32_t crow_s = uint32_t(__cvta_generic_to_shared(codes)) + uint32_t(tid) * cstride;
  RowMap rm;
  rm.HD = uint64_t(H) * D;
  rm.rows = rows;
  rm.row0 = PAGED ? nullptr : dest_row(p, chunk, slab, n, s_tstart, unit_t0);
  const int DS = D / kSlices;  // channels of a slice (a multiple of 8)
  const int dq = kThreads / (DS >> 3), dr = kThreads - dq * (DS >> 3);
  __syncthreads();
  if (tid < ngroups) {  // whole-group flags for phase B's fast path
    const int t0 = tid * kGroup, t1 = min(t0 + kGroup, ntok);
    int all = 1;
    for (int t = t0; t < t1; ++t) all &= okf[t];
    gok[tid] = uint8_t(all);
  }

  for (int h = 0; h < H; ++h) {
    for (int sl = 0; sl < kSlices; ++sl) {
      const bool last = sl == kSlices - 1;
      // ---- phase A: the codes of slice sl of head h
      if (active) {
        const int one = single[h];
        if (one >= 0) {  // a one-symbol table: the state stays put, no word is read
          const uint32_t cc = uint32_t(one) * 0x01010101u;
          for (int d0 = 0; d0 < DS; d0 += 8)
            asm volatile("st.shared.v2.u32 [%0], {%1, %1};\n" ::"r"(crow_s + uint32_t(d0)), "r"(cc)
                         : "memory");
        } else {
          decode_codes(x, pw, ra, w, ring, tbl_s, crow_s, DS);
        }
      }
      // global loads for the next heads are issued before the barrier
      const bool scan_warp = last && h + 2 < H && warp == h % kWarps;
      uint4 fq = make_uint4(0, 0, 0, 0);
      if (scan_warp) fq = __ldg(reinterpret_cast<const uint4*>(freq + (h + 2) * 256) + lane);
      float zv[2] = {0.0f, 0.0f};
      const bool stage = last && h + 1 < H;
      if (stage) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int i = tid + j * kThreads;
          if (i < 2 * D)
            zv[j] = i < D ? __ldg(zp_sec + (h + 1) * D + i) : __ldg(sc_sec + (h + 1) * D + (i - D));
        }
      }
      __syncthreads();
      // ---- phase B: fp16 values of slice sl of head h; after the last slice
      // the table, zero points and scales of head h + 1 and the compacted
      // table of head h + 2
      dequant_head<ADJ, PAGED>(codes, cstride, zs + (h & 1) * 2 * D, rm, okf, gok, ngroups, ntok,
                               h, D, sl * DS, DS, step, tid, dq, dr);
      if (stage) {
        // phase A of head h is over: the table is rebuilt for head h + 1
        fill_table(tbl, cum_buf(cumb + ((h + 1) & 1) * kCumBuf), tid);
        float* zn = zs + ((h + 1) & 1) * 2 * D;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int i = tid + j * kThreads;
          if (i < 2 * D) zn[i] = zv[j];
        }
      }
      if (scan_warp) cum_compact(fq, cum_buf(cumb + (h & 1) * kCumBuf), lane);
      __syncthreads();
    }
  }
  ring_wait_all();
  if (active && (x != kRansL || pw != pend)) set_status(p.status, CG_ERR_CORRUPT);
}

}  // namespace

cudaError_t launch_decode(const DecParams& p, cudaStream_t stream) {
  const DecSmem sm = dec_smem(p.H, p.D);
  auto* kern = p.adjacent ? (p.into == 2 ? decode_kernel<true, true> : decode_kernel<true, false>)
                          : (p.into == 2 ? decode_kernel<false, true> : decode_kernel<false, false>);
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm.total));
  if (err != cudaSuccess) return err;
  const uint64_t blocks = uint64_t(p.num_chunks) * p.L * 2 * p.units_per_slab;
  kern<<<unsigned(blocks), kThreads, sm.total, stream>>>(p);
  return cudaGetLastError();
}

int decode_units_per_slab(int C) {
  const int groups = (C + kGroup - 1) / kGroup;
  return (groups + kUnitGroups - 1) / kUnitGroups;
}

}  // namespace cg
