// encode.cu -- the CacheGen encoder: anchor range, anchor + delta quantiser
// with per-head histograms and 12-bit table normalisation, rANS encoding of
// one stream per (layer, K/V, token), the stream-offset prefix sum, and the
// compaction of the streams into the container payload.
//
// [Practice] 1: quantise the difference to nearby tokens with a layer-wise
// step, then entropy-code ("grouped entropy coding"); [Practice] 2.1: every
// chunk is encoded on its own; [Practice] 3.1: the step tables; [Overview]
// KV-cache quantisation mechanism: per-channel scale and zero point.
//
// Kernels, in launch order:
//   quant_kernel    one CTA per (chunk, l, kv, h): anchor range -> zp, scale;
//                   anchor codes and reconstructed anchors; delta symbols;
//                   lane-replicated shared histogram; frequency table and the
//                   encoder's per-symbol division constants.  quant_kernel<3>
//                   (cg_encode_levels) quantises every delta at the three
//                   levels' steps from one read and keeps three histograms;
//                   the three kernels below then run once per level.
//   rans_kernel     one thread per stream (l, kv, t), symbols in reverse;
//                   renormalisation words go through a per-thread ring in
//                   shared memory and leave in 32-byte blocks, written
//                   backwards into a per-stream scratch slot.
//   offsets_kernel  one CTA per (chunk, layer, K/V): its base (the words of the
//                   earlier layers, summed by the rANS pass) plus an exclusive
//                   scan of its stream lengths -> offsets; the last one of a
//                   chunk writes the header and the container size.
//   compact_kernel  one warp per stream: scratch slot -> payload.
//
// A call of two or more chunks runs this sequence twice, once per half of its
// chunks, the second half on the library's side stream (launch_encode).
#include <cuda_fp16.h>

#include "cg_common.cuh"

namespace cg {
namespace {

constexpr int kQThreads = 256;
constexpr int kQWarps = kQThreads / 32;
constexpr int kRThreads = 128;                     // rANS streams per CTA
constexpr int kRing = 64;                          // u16 ring entries per thread
constexpr int kRingStride = 72;                    // u16; 144 B keeps 16-B alignment and
                                                   // staggers the threads' banks
constexpr int kScanThreads = 256;

enum QuantMode { kModeEncode = 0, kModeTablesOnly = 1, kModeSuppliedTables = 2 };

// Shared memory of quant_kernel<NL> (NL = levels quantised at once: 1, or 3
// for the three-level encoder).
struct QSmem {
  uint32_t hist;    // u32 [NL][255][32]  lane-replicated counters (bank = lane)
  uint32_t zp;      // f32 [256]
  uint32_t sc;      // f32 [256]
  uint32_t rcp;     // f32 [256]
  uint32_t red;     // f32 [2][8 warps][256]  anchor range partials (phase A)
  uint32_t counts;  // u32 [NL][256]  histogram totals (phase C)
  uint32_t total;
};

__host__ __device__ inline uint32_t a16(uint32_t v) { return (v + 15u) & ~15u; }

template <int NL>
__host__ __device__ inline QSmem q_smem() {
  QSmem s;
  s.hist = 0;
  s.zp = a16(s.hist + NL * 255u * 32u * 4u);
  s.sc = s.zp + 1024u;
  s.rcp = s.sc + 1024u;
  if (NL == 1) {
    s.red = s.rcp + 1024u;
    s.counts = s.red;  // phase C reuses the phase-A partials
    s.total = a16(s.red + 2u * kQWarps * 256u * 4u);
  } else {
    // The phase-A partials live in the histogram space, which is cleared
    // after phase A; two CTAs per SM still fit.
    s.red = s.hist;
    s.counts = s.rcp + 1024u;
    s.total = a16(s.counts + NL * 256u * 4u);
  }
  return s;
}

// Count the symbol of bracket word t = 0x4B400000 + u in the lane's column of
// the shared histogram: hb is the column's address minus 0xA0000000, since
// t << 7 = 0xA0000000 + 128 u modulo 2^32.
__device__ __forceinline__ void hist_add(uint32_t hb, uint32_t t) {
  asm volatile("red.shared.add.u32 [%0], 1;\n" ::"r"(hb + (t << 7)) : "memory");
}

// Exact quantisation of d = x - a by a step s with precomputed r = RN(1/s).
// y = RN(d * r) is within 3 * 2^-24 |y| of RN(d / s) (three roundings of
// relative size 2^-24).  The two values yc (1 - 2^-20) and yc (1 + 2^-20), yc
// = y clamped to [-127, 127], bracket RN(d / s) (clamped alike) with room to
// spare; each is rounded to an integer by one fused add of 1.5 * 2^23 + 127
// (ulp 1 there), giving the word t = 0x4B400000 + u.  When both give the same
// integer, no half-integer lies between them, so round-half-away-from-zero of
// RN(d / s) gives that integer too.  For a row of 8 values the caller ORs
// t1 ^ t2 into `diff` and takes the definition (quant_exact) for the whole row
// when any bit differs.  A quotient that is not finite (an infinite or NaN
// input) cannot be bracketed: y * 0 turns `nanacc` into NaN, and the caller
// reports the input.  Every finite y is clamped into [-127, 127], where the
// bracket holds (a huge quotient clamps to +-127 on both paths).
__device__ __forceinline__ uint32_t quant_bits(float d, float r, uint32_t& diff, float& nanacc) {
  const float y = __fmul_rn(d, r);
  nanacc = __fmaf_rn(y, 0.0f, nanacc);
  const float yc = fminf(fmaxf(y, -127.0f), 127.0f);
  const uint32_t t1 = __float_as_uint(__fmaf_rn(yc, 1.0f + 0x1p-20f, 12583039.0f));
  const uint32_t t2 = __float_as_uint(__fmaf_rn(yc, 1.0f - 0x1p-20f, 12583039.0f));
  diff |= t1 ^ t2;
  return t1;
}

// The definition itself: u = clamp(roundf(RN(RN(x - a) / s)), -127, 127) + 127,
// with s == 0 (a constant anchor channel) giving code 0; returned in the form
// of a bracket word, 0x4B400000 + u.
__device__ __forceinline__ uint32_t quant_exact(float x, float a, float s) {
  if (s == 0.0f) return 0x4B400000u + 127u;
  const float y = __fdiv_rn(__fsub_rn(x, a), s);
  const float r = fminf(fmaxf(roundf(y), -127.0f), 127.0f);
  return 0x4B400000u + uint32_t(int(r) + 127);
}

// (float)q of a bracket word t = 0x4B400000 + u: t is the float 2^23 + 2^22 + u,
// and subtracting 2^23 + 2^22 + 127 is exact.
__device__ __forceinline__ float code_of(uint32_t t) {
  return __fsub_rn(__uint_as_float(t), 12583039.0f);
}

__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t v) {
  return __reduce_add_sync(0xFFFFFFFFu, v);
}
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
  return __reduce_max_sync(0xFFFFFFFFu, v);
}

// Normalise the 255 counts of one table to frequencies summing to 4096 (the
// rule stated in cachegen.h).  One warp; lane holds u = 8 lane + i.  The
// "decrement the largest" loop is applied level by level: all symbols tied at
// the current maximum drop together to the next distinct value, and a final
// partial round takes the tied symbols in increasing u order, which is what
// the one-at-a-time rule does.
__device__ void normalize_warp(const uint32_t* counts, uint64_t N, uint32_t f[8], int lane) {
  uint32_t c[8];
  uint32_t sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int u = lane * 8 + i;
    c[i] = u < kAlphabet ? counts[u] : 0u;
    uint32_t v = 0;
    if (c[i]) {
      v = uint32_t((uint64_t(c[i]) * kM) / N);
      if (v < 1) v = 1;
    }
    f[i] = v;
    sum += v;
  }
  sum = warp_sum_u32(sum);
  if (sum < kM) {
    // Largest count, ties to the smallest u: maximise (count, 255 - u).
    unsigned long long key = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int u = lane * 8 + i;
      if (c[i]) {
        const unsigned long long k = (static_cast<unsigned long long>(c[i]) << 8) | uint32_t(255 - u);
        key = k > key ? k : key;
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xFFFFFFFFu, key, o);
      key = other > key ? other : key;
    }
    const int best = 255 - int(key & 0xFF);
    if ((best >> 3) == lane) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (i == (best & 7)) f[i] += kM - sum;
    }
    return;
  }
  uint32_t excess = sum - kM;
  while (excess > 0) {
    uint32_t m1 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (f[i] > 1 && f[i] > m1) m1 = f[i];
    m1 = warp_max_u32(m1);
    if (m1 == 0) break;  // unreachable: 255 ones sum to less than 4096
    uint32_t tied = 0, m2 = 1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (f[i] == m1) ++tied;
      else if (f[i] < m1 && f[i] > m2) m2 = f[i];
    }
    const uint32_t c1 = warp_sum_u32(tied);
    m2 = warp_max_u32(m2);
    if (uint64_t(c1) * (m1 - m2) <= excess) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (f[i] == m1) f[i] = m2;
      excess -= c1 * (m1 - m2);
    } else {
      const uint32_t full = excess / c1, extra = excess % c1;
      uint32_t rank = tied;  // exclusive prefix of tied counts over lanes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, rank, o);
        if (lane >= o) rank += v;
      }
      rank -= tied;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (f[i] == m1) {
          f[i] -= full + (rank < extra ? 1u : 0u);
          ++rank;
        }
      }
      excess = 0;
    }
  }
}

// Encoder constants of one symbol.  The state stays in [2^15, 2^31), so
// floor(x / f) = umulhi(2x, m) >> l with l = ceil(log2 f) and the 32-bit
// multiplier m = ceil(2^(31+l) / f) (Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994, theorem 4.2 with N = 31).
//   .x = (f << 19) - 1   the largest state that needs no renormalisation
//   .y = m
//   .z = cum
//   .w = ((4096 - f) << 5) | l   (a funnel shift reads l from the low 5 bits)
// Sixteen bytes per entry keep the per-symbol arithmetic minimal; an absent
// symbol (f == 0) gets .w = 0xFFFFFFFF, which no present symbol has.
__device__ __forceinline__ uint4 enc_entry(uint32_t f, uint32_t cum) {
  if (f == 0) return make_uint4(0xFFFFFFFFu, 0u, 0u, 0xFFFFFFFFu);
  const uint32_t lg = f == 1 ? 0u : 32u - __clz(f - 1);  // ceil(log2 f)
  const uint64_t num = 1ull << (31 + lg);
  const uint32_t magic = uint32_t((num + f - 1) / f);
  return make_uint4((f << 19) - 1u, magic, cum, ((kM - f) << 5) | lg);
}

// Lane layout of the quantiser: a lane covers 8 channels (one 16-byte load of
// a token's head row); D/8 lanes cover a row, so a warp covers rpw = 32/(D/8)
// rows at once and works on rpw anchor groups side by side (lane row r takes
// group gs * rpw + r of group set gs).
struct QLanes {
  int lpr, rpw, r, c;
  bool on;
};

__device__ __forceinline__ QLanes q_lanes(int D, int lane) {
  QLanes q;
  q.lpr = D / 8;
  q.rpw = 32 / q.lpr;
  q.r = lane / q.lpr;
  q.c = lane - q.r * q.lpr;
  q.on = q.r < q.rpw;
  return q;
}

__device__ __forceinline__ void unpack8(const uint4 rv, float (&x)[8]) {
  const uint32_t raw[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&raw[q]));
    x[2 * q] = f2.x;
    x[2 * q + 1] = f2.y;
  }
}

// quant_kernel<NL, ADJ>: NL = 1 quantises at the call's level (cg_encode,
// cg_build_tables); NL = 3 quantises every delta at the three levels' steps
// from one read of the fp16 rows (cg_encode_levels: [Practice] 2.1 keeps three
// versions of every chunk).  The anchor range, the anchor codes and the
// reconstructed anchors do not depend on the level, so they are computed once
// and the anchor codes enter every level's streams and histogram.
// ADJ (format 2, cg_encode_adjacent): each delta is taken against the
// reconstruction of the token before it ([Practice] 1: differences between
// adjacent tokens) instead of the group's anchor; a lane walks its group's
// rows in order, so the running reconstruction stays in its registers.
template <int NL, bool ADJ>
__global__ void __launch_bounds__(kQThreads, NL == 1 ? 3 : 2) quant_kernel(const EncParams p, const int mode) {
  static_assert(!(ADJ && NL != 1), "format 2 is encoded one level at a time");
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int rest = blockIdx.x;
  const int h = rest % p.H;
  rest /= p.H;
  const int kv = rest & 1;
  rest >>= 1;
  const int l = rest % p.L;
  const int chunk = rest / p.L;
  const int L = p.L, H = p.H, D = p.D, C = p.C;
  const int64_t t0 = p.token_start + int64_t(chunk) * C;
  const int n = int(min(int64_t(C), p.T - t0));
  const int Gn = (n + kGroup - 1) / kGroup;
  const int slab = l * 2 + kv;
  const int tab = slab * H + h;
  const uint64_t rs = uint64_t(H) * D;
  const uint16_t* col = p.kv + (uint64_t(slab) * p.T + t0) * rs + uint64_t(h) * D;

  const QSmem sm = q_smem<NL>();
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + sm.hist);
  float* zp = reinterpret_cast<float*>(smem + sm.zp);
  float* sc = reinterpret_cast<float*>(smem + sm.sc);
  float* rcp = reinterpret_cast<float*>(smem + sm.rcp);
  float* red = reinterpret_cast<float*>(smem + sm.red);
  uint32_t* counts = reinterpret_cast<uint32_t*>(smem + sm.counts);

  const Sections sec = sections(L, H, D, n);
  // container of level j (of the call's level when NL == 1)
  auto cont_of = [&](int j) -> uint8_t* {
    uint8_t* o = NL == 1 ? p.out : p.lout[j];
    return o ? o + uint64_t(chunk) * p.out_stride : nullptr;
  };
  // Table block offsets equal container offsets minus the header.
  const uint64_t tb_zp = sec.zp - CG_HEADER_BYTES, tb_sc = sec.scale - CG_HEADER_BYTES,
                 tb_fq = sec.freq - CG_HEADER_BYTES;
  const bool want_hist = mode != kModeSuppliedTables;
  const bool want_sym = mode != kModeTablesOnly;
  const QLanes ql = q_lanes(D, lane);
  const int ch = 8 * ql.c;  // first channel of this lane
  const int nsets = (Gn + ql.rpw - 1) / ql.rpw;

  if (NL == 1 && want_hist)
    for (int i = tid; i < kAlphabet * 32; i += kQThreads) hist[i] = 0;
  if (want_sym && h == 0 && tid == 0) {
#pragma unroll
    for (int j = 0; j < NL; ++j)
      (NL == 1 ? p.slabtot : p.lslabtot[j])[uint64_t(chunk) * L * 2 + slab] = 0;
  }

  // ---- Phase A: per-channel anchor range -> zp, scale (or the supplied ones).
  bool nonfinite = false;
  if (mode == kModeSuppliedTables) {
    const uint8_t* tb = p.tables_in + uint64_t(chunk) * p.tables_stride;
    for (int d = tid; d < D; d += kQThreads) {
      zp[d] = reinterpret_cast<const float*>(tb + tb_zp)[uint64_t(tab) * D + d];
      sc[d] = reinterpret_cast<const float*>(tb + tb_sc)[uint64_t(tab) * D + d];
    }
  } else {
    float lo[8], hi[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      lo[k] = __int_as_float(0x7F800000);
      hi[k] = -lo[k];
    }
    for (int gs = warp; gs < nsets; gs += 4 * kQWarps) {  // four anchor rows in flight
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int g = (gs + j * kQWarps) * ql.rpw + ql.r;
        v[j] = ql.on && g < Gn
                   ? __ldg(reinterpret_cast<const uint4*>(col + uint64_t(g) * kGroup * rs + ch))
                   : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int g = (gs + j * kQWarps) * ql.rpw + ql.r;
        if (!(ql.on && g < Gn)) continue;
        float x[8];
        unpack8(v[j], x);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (!isfinite(x[k])) nonfinite = true;
          lo[k] = fminf(lo[k], x[k]);
          hi[k] = fmaxf(hi[k], x[k]);
        }
      }
    }
    // partials of (warp, lane row) -> red[{lo, hi}][warp * rpw + r][channel]
    if (ql.on) {
      float* rl = red + (warp * ql.rpw + ql.r) * D + ch;
      float* rh = rl + kQWarps * 256;
      *reinterpret_cast<float4*>(rl) = make_float4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<float4*>(rl + 4) = make_float4(lo[4], lo[5], lo[6], lo[7]);
      *reinterpret_cast<float4*>(rh) = make_float4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<float4*>(rh + 4) = make_float4(hi[4], hi[5], hi[6], hi[7]);
    }
    __syncthreads();
    for (int d = tid; d < D; d += kQThreads) {
      float lo1 = red[d], hi1 = red[kQWarps * 256 + d];
      for (int j = 1; j < kQWarps * ql.rpw; ++j) {
        lo1 = fminf(lo1, red[j * D + d]);
        hi1 = fmaxf(hi1, red[kQWarps * 256 + j * D + d]);
      }
      zp[d] = __fmul_rn(__fadd_rn(lo1, hi1), 0.5f);
      sc[d] = __fdiv_rn(__fsub_rn(hi1, lo1), 254.0f);
    }
  }
  __syncthreads();
  if (NL > 1 && want_hist)  // the phase-A partials are consumed: clear the histograms
    for (int i = tid; i < NL * kAlphabet * 32; i += kQThreads) hist[i] = 0;
  for (int d = tid; d < D; d += kQThreads) {
    rcp[d] = sc[d] == 0.0f ? 0.0f : __frcp_rn(sc[d]);
#pragma unroll
    for (int j = 0; j < NL; ++j) {
      uint8_t* cont = cont_of(j);
      if (cont) {
        reinterpret_cast<float*>(cont + sec.zp)[uint64_t(tab) * D + d] = zp[d];
        reinterpret_cast<float*>(cont + sec.scale)[uint64_t(tab) * D + d] = sc[d];
      }
    }
    if (p.tables_out) {
      uint8_t* tb = p.tables_out + uint64_t(chunk) * p.tables_stride;
      reinterpret_cast<float*>(tb + tb_zp)[uint64_t(tab) * D + d] = zp[d];
      reinterpret_cast<float*>(tb + tb_sc)[uint64_t(tab) * D + d] = sc[d];
    }
  }
  __syncthreads();

  // ---- Phase B: quantise group by group.  A lane walks the ten rows of its
  // group for its 8 channels (one 16-byte load per row), then the ten rows of
  // its next group set; the loads run five rows ahead in a register ring,
  // across the boundary between group sets.
  float step[NL], rstep[NL];
#pragma unroll
  for (int j = 0; j < NL; ++j) {
    step[j] = step_of(NL == 1 ? p.level : j, l, L);
    rstep[j] = __frcp_rn(step[j]);
  }
  const uint64_t symo = ((uint64_t(chunk) * L * 2 + slab) * H + h) * uint64_t(D / 16) * C * 16 +
                        (ql.c >> 1) * uint64_t(C) * 16 + (ql.c & 1) * 8;
  auto symc_of = [&](int j) { return (NL == 1 ? p.sym : p.lsym[j]) + symo; };
  // Histogram counter of symbol u for this lane: hist + 4 lane + 128 u (bank =
  // lane).  A bracket word is t = 0x4B400000 + u (see quant_bits), so
  // t << 7 = 0xA0000000 + 128 u modulo 2^32 and the address is one shift-add.
  const uint32_t hist_t = uint32_t(__cvta_generic_to_shared(hist)) + 4u * lane - 0xA0000000u;
  auto put_syms = [&](int j, int tok, uint32_t t0, uint32_t t1, uint32_t t2, uint32_t t3,
                      uint32_t t4, uint32_t t5, uint32_t t6, uint32_t t7) {
    if (want_hist) {
      const uint32_t hb = hist_t + (uint32_t(j * kAlphabet) << 7);
      hist_add(hb, t0);
      hist_add(hb, t1);
      hist_add(hb, t2);
      hist_add(hb, t3);
      hist_add(hb, t4);
      hist_add(hb, t5);
      hist_add(hb, t6);
      hist_add(hb, t7);
    }
    if (want_sym)
      *reinterpret_cast<uint2*>(symc_of(j) + uint64_t(tok) * 16) =
          make_uint2(__byte_perm(__byte_perm(t0, t1, 0x0040), __byte_perm(t2, t3, 0x0040), 0x5410),
                     __byte_perm(__byte_perm(t4, t5, 0x0040), __byte_perm(t6, t7, 0x0040), 0x5410));
  };
  // rows of group set gs available to this lane (0 past the chunk's groups)
  auto set_rows = [&](int gs) {
    const int g = gs * ql.rpw + ql.r;
    return (ql.on && gs < nsets && g < Gn) ? min(kGroup, n - g * kGroup) : 0;
  };
  auto set_ptr = [&](int gs) {
    return col + uint64_t(gs * ql.rpw + ql.r) * kGroup * rs + ch;
  };
  float nanacc = 0.0f;  // becomes NaN once a quotient is not finite
  constexpr int kAhead = 5;  // ring depth (kGroup is a multiple of it)
  uint4 ring[kAhead];
  int ntok = set_rows(warp);
  const uint16_t* rp = set_ptr(warp);
#pragma unroll
  for (int j = 0; j < kAhead; ++j)
    ring[j] = j < ntok ? __ldg(reinterpret_cast<const uint4*>(rp + uint64_t(j) * rs))
                       : make_uint4(0, 0, 0, 0);
  for (int gs = warp; gs < nsets; gs += kQWarps) {
    const int tg = (gs * ql.rpw + ql.r) * kGroup;
    const int ntok_next = set_rows(gs + kQWarps);
    const uint16_t* rpn = set_ptr(gs + kQWarps);
    float a[8];
#pragma unroll
    for (int r = 0; r < kGroup; ++r) {
      const uint4 cur = ring[r % kAhead];
      // refill the slot: row r + 5 of this set, or row r - 5 of the next one
      if (r + kAhead < kGroup) {
        ring[r % kAhead] = r + kAhead < ntok
            ? __ldg(reinterpret_cast<const uint4*>(rp + uint64_t(r + kAhead) * rs))
            : make_uint4(0, 0, 0, 0);
      } else {
        ring[r % kAhead] = r + kAhead - kGroup < ntok_next
            ? __ldg(reinterpret_cast<const uint4*>(rpn + uint64_t(r + kAhead - kGroup) * rs))
            : make_uint4(0, 0, 0, 0);
      }
      if (r >= ntok) continue;
      float x[8];
      unpack8(cur, x);
      if (r == 0) {
        // anchor: code against (zp, scale), reconstructed value a
        float zc[8], scc[8], rc[8];
#pragma unroll
        for (int k = 0; k < 8; k += 4) {  // this lane's channels, from shared memory
          const float4 za = *reinterpret_cast<const float4*>(zp + ch + k);
          const float4 sa = *reinterpret_cast<const float4*>(sc + ch + k);
          const float4 ra = *reinterpret_cast<const float4*>(rcp + ch + k);
          zc[k] = za.x; zc[k + 1] = za.y; zc[k + 2] = za.z; zc[k + 3] = za.w;
          scc[k] = sa.x; scc[k + 1] = sa.y; scc[k + 2] = sa.z; scc[k + 3] = sa.w;
          rc[k] = ra.x; rc[k + 1] = ra.y; rc[k + 2] = ra.z; rc[k + 3] = ra.w;
        }
        uint32_t t[8], diff = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) t[k] = quant_bits(__fsub_rn(x[k], zc[k]), rc[k], diff, nanacc);
        if (diff) {
#pragma unroll
          for (int k = 0; k < 8; ++k) t[k] = quant_exact(x[k], zc[k], scc[k]);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) a[k] = __fadd_rn(zc[k], __fmul_rn(code_of(t[k]), scc[k]));
#pragma unroll
        for (int j = 0; j < NL; ++j) put_syms(j, tg, t[0], t[1], t[2], t[3], t[4], t[5], t[6], t[7]);
      } else {
#pragma unroll
        for (int j = 0; j < NL; ++j) {
          uint32_t t[8], diff = 0;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            t[k] = quant_bits(__fsub_rn(x[k], a[k]), rstep[j], diff, nanacc);
          if (diff) {
#pragma unroll
            for (int k = 0; k < 8; ++k) t[k] = quant_exact(x[k], a[k], step[j]);
          }
          put_syms(j, tg + r, t[0], t[1], t[2], t[3], t[4], t[5], t[6], t[7]);
          if (ADJ) {  // the next row's reference: this row's reconstruction
#pragma unroll
            for (int k = 0; k < 8; ++k) a[k] = __fadd_rn(a[k], __fmul_rn(code_of(t[k]), step[j]));
          }
        }
      }
    }
    ntok = ntok_next;
    rp = rpn;
  }
  if (nanacc != nanacc) nonfinite = true;
  __syncthreads();
  if (nonfinite) set_status(p.status, CG_ERR_NONFINITE);

  // ---- Phase C: histograms -> frequency tables -> encoder constants (warp j
  // normalises level j's table).
  if (want_hist) {
    for (int i = tid; i < NL * kAlphabet; i += kQThreads) {
      const int j = i / kAlphabet, u = i - j * kAlphabet;
      const uint32_t* hj = hist + j * kAlphabet * 32;
      uint32_t s = 0;
      for (int r = 0; r < 32; ++r) s += hj[u * 32 + ((r + u) & 31)];
      counts[j * 256 + u] = s;
    }
    __syncthreads();
  }
  if (warp < NL) {
    const int j = warp;
    uint32_t f[8];
    if (mode == kModeSuppliedTables) {
      const uint16_t* fq = reinterpret_cast<const uint16_t*>(
          p.tables_in + uint64_t(chunk) * p.tables_stride + tb_fq) + uint64_t(tab) * 256;
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = fq[lane * 8 + i];
    } else {
      normalize_warp(counts + j * 256, uint64_t(n) * D, f, lane);
    }
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) pk[i] = f[2 * i] | (f[2 * i + 1] << 16);
    const uint4 fv = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    uint8_t* cont = cont_of(j);
    if (cont)
      reinterpret_cast<uint4*>(cont + sec.freq + uint64_t(tab) * 512)[lane] = fv;
    if (p.tables_out)
      reinterpret_cast<uint4*>(p.tables_out + uint64_t(chunk) * p.tables_stride + tb_fq +
                               uint64_t(tab) * 512)[lane] = fv;
    if (want_sym) {
      uint32_t local = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) local += f[i];
      uint32_t incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
      }
      uint32_t cum = incl - local;
      uint4* et = reinterpret_cast<uint4*>(NL == 1 ? p.etab : p.letab[j]) +
                  ((uint64_t(chunk) * L * 2 + slab) * H + h) * 256;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        et[lane * 8 + i] = enc_entry(f[i], cum & 0xFFFF);
        cum += f[i];
      }
    }
  }
}

__device__ __forceinline__ uint32_t swap16(uint32_t v) { return __byte_perm(v, 0, 0x1032); }

// One rANS encoder step with the constants e of the symbol (see enc_entry):
// renormalise by pushing the low 16 bits into the thread's ring when
// x > (f << 19) - 1, then x = floor(x / f) * 4096 + x mod f + cum computed as
// x + cum + q * (4096 - f).  Predicated rather than branched; the asm does not
// clobber memory, so the caller orders the ring reads with a compiler barrier.
__device__ __forceinline__ void enc_step(uint32_t& x, uint32_t& wp, uint32_t ring_s,
                                         const uint4& e) {
  asm volatile(
      "{\n\t"
      ".reg .pred p;\n\t"
      ".reg .u32 a, t, q;\n\t"
      "setp.gt.u32 p, %0, %3;\n\t"
      "@p and.b32 a, %1, 63;\n\t"
      "@p mad.lo.u32 a, a, 2, %2;\n\t"
      "@p st.shared.u16 [a], %0;\n\t"
      "@p add.u32 %1, %1, 1;\n\t"
      "@p shr.u32 %0, %0, 16;\n\t"
      "add.u32 t, %0, %0;\n\t"
      "mul.hi.u32 t, t, %4;\n\t"
      "shf.r.wrap.b32 q, t, 0, %6;\n\t"
      "shr.u32 t, %6, 5;\n\t"
      "add.u32 %0, %0, %5;\n\t"
      "mad.lo.u32 %0, q, t, %0;\n\t"
      "}\n"
      : "+r"(x), "+r"(wp)
      : "r"(ring_s), "r"(e.x), "r"(e.y), "r"(e.z), "r"(e.w));
}

template <bool kCheckF>
__global__ void __launch_bounds__(kRThreads, 6) rans_kernel(const EncParams p) {
  __shared__ __align__(16) uint4 et[2][256];
  __shared__ __align__(16) uint16_t ring[kRThreads * kRingStride];
  const int tid = threadIdx.x;
  const int C = p.C, L = p.L, H = p.H, D = p.D;
  const int tiles = (C + kRThreads - 1) / kRThreads;
  const int tile = blockIdx.x % tiles;
  int rest = blockIdx.x / tiles;
  const int slab = rest % (2 * L);
  const int chunk = rest / (2 * L);
  const int64_t t0 = p.token_start + int64_t(chunk) * C;
  const int n = int(min(int64_t(C), p.T - t0));
  if (tile * kRThreads >= n) return;
  const int t = tile * kRThreads + tid;
  const bool active = t < n;
  const int nb = D / 16;
  const uint64_t cs = uint64_t(chunk) * L * 2 + slab;
  const uint4* etg = reinterpret_cast<const uint4*>(p.etab) + cs * H * 256;
  // symbols of this token, 16-byte blocks ordered (h, b); block index h*nb + b
  const uint4* symt = reinterpret_cast<const uint4*>(p.sym + cs * H * uint64_t(nb) * C * 16) + t;
  const uint64_t ss = scratch_stride(H, D);
  uint16_t* rend = active ? reinterpret_cast<uint16_t*>(p.scratch + (cs * C + t + 1) * ss) : nullptr;
  uint16_t* myring = ring + tid * kRingStride;
  const uint32_t ring_s = uint32_t(__cvta_generic_to_shared(myring));

  // Stage the last head's encoder table; prefetch the next one into registers.
  et[(H - 1) & 1][tid] = __ldg(etg + uint64_t(H - 1) * 256 + tid);
  et[(H - 1) & 1][tid + kRThreads] = __ldg(etg + uint64_t(H - 1) * 256 + tid + kRThreads);
  uint32_t x = kRansL, wp = 0, wf = 0;
  bool bad = false;
  int blk = H * nb - 1;  // next 16-symbol block, walking backwards
  // symbol blocks are loaded two blocks (32 symbols) ahead of their use
  uint4 vnext = active ? __ldg(symt + uint64_t(blk) * C) : make_uint4(0, 0, 0, 0);
  uint4 vnext2 = active && blk > 0 ? __ldg(symt + uint64_t(blk - 1) * C) : make_uint4(0, 0, 0, 0);
  for (int h = H - 1; h >= 0; --h) {
    uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
    if (h > 0) {
      n0 = __ldg(etg + uint64_t(h - 1) * 256 + tid);
      n1 = __ldg(etg + uint64_t(h - 1) * 256 + tid + kRThreads);
    }
    __syncthreads();  // table h is staged; nobody reads buffer (h+1)&1 any more
    const uint4* eh = et[h & 1];
    if (active) {
      for (int b = nb - 1; b >= 0; --b, --blk) {
        const uint4 v = vnext;
        vnext = vnext2;
        if (blk > 1) vnext2 = __ldg(symt + uint64_t(blk - 2) * C);
#pragma unroll
        for (int k = 15; k >= 0; --k) {
          const uint32_t word = (k >> 2) == 0 ? v.x : (k >> 2) == 1 ? v.y : (k >> 2) == 2 ? v.z : v.w;
          const uint32_t u = (word >> (8 * (k & 3))) & 0xFFu;
          const uint4 e = eh[u];
          enc_step(x, wp, ring_s, e);
          if (kCheckF) bad |= e.w == 0xFFFFFFFFu;
        }
        // the ring stores inside enc_step precede the ring reads of the flush
        asm volatile("" ::: "memory");
        if (wp - wf >= 16) {
          const uint4* src = reinterpret_cast<const uint4*>(myring + (wf & (kRing - 1)));
          const uint4 r0 = src[0], r1 = src[1];
          // one 256-bit store (a full L2 sector; rend - wf - 16 is 32-byte aligned)
          uint16_t* dst = rend - wf - 16;
          asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"l"(dst),
                       "r"(swap16(r1.w)), "r"(swap16(r1.z)), "r"(swap16(r1.y)), "r"(swap16(r1.x)),
                       "r"(swap16(r0.w)), "r"(swap16(r0.z)), "r"(swap16(r0.y)), "r"(swap16(r0.x))
                       : "memory");
          wf += 16;
        }
      }
    }
    if (h > 0) {
      et[(h - 1) & 1][tid] = n0;
      et[(h - 1) & 1][tid + kRThreads] = n1;
    }
  }
  asm volatile("" ::: "memory");
  if (active) {
    myring[wp & (kRing - 1)] = uint16_t(x);
    ++wp;
    myring[wp & (kRing - 1)] = uint16_t(x >> 16);
    ++wp;
    for (uint32_t k = wf; k < wp; ++k) rend[-1 - int64_t(k)] = myring[k & (kRing - 1)];
    p.lens[cs * C + t] = wp;
    if (kCheckF && bad) set_status(p.status, CG_ERR_MISMATCH);
  }
  // this CTA's share of the (layer, K/V) total, for the offsets pass
  const uint32_t mine = __reduce_add_sync(0xFFFFFFFFu, active ? wp : 0u);
  if ((tid & 31) == 0) atomicAdd(p.slabtot + cs, mine);
}

// Block-wide exclusive scan of one value per thread (kScanThreads threads).
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tot,
                                                         uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t t = lane < kScanThreads / 32 ? warp_tot[lane] : 0u;
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, ti, o);
      if (lane >= o) ti += u;
    }
    if (lane < kScanThreads / 32) warp_tot[lane] = ti - t;
    if (lane == 31) warp_tot[32] = ti;
  }
  __syncthreads();
  total = warp_tot[32];
  return warp_tot[warp] + incl - v;
}

// One CTA per (chunk, layer, K/V): the offsets of its streams are the words of
// every earlier (layer, K/V) of the chunk plus an exclusive scan of its own
// stream lengths.  The last (layer, K/V) of a chunk also writes the header.
__global__ void __launch_bounds__(kScanThreads) offsets_kernel(const EncParams p) {
  __shared__ uint32_t warp_tot[33];
  const int tid = threadIdx.x;
  const int C = p.C, L = p.L, H = p.H, D = p.D;
  const int slab = blockIdx.x % (2 * L);
  const int chunk = blockIdx.x / (2 * L);
  const int64_t t0 = p.token_start + int64_t(chunk) * C;
  const int n = int(min(int64_t(C), p.T - t0));
  const Sections sec = sections(L, H, D, n);
  uint8_t* cont = p.out + uint64_t(chunk) * p.out_stride;
  uint32_t* offs = reinterpret_cast<uint32_t*>(cont + sec.offsets) + uint64_t(slab) * n;
  const uint32_t* tot = p.slabtot + uint64_t(chunk) * L * 2;
  const uint32_t* lens = p.lens + (uint64_t(chunk) * L * 2 + slab) * C;

  uint32_t part = 0;
  for (int i = tid; i < slab; i += kScanThreads) part += tot[i];
  uint32_t base_total;
  block_exclusive_scan(part, warp_tot, base_total);  // only the total is used
  const uint32_t base = base_total;
  __syncthreads();  // warp_tot is reused below

  const int per = (n + kScanThreads - 1) / kScanThreads;
  const int s0 = min(n, tid * per), s1 = min(n, s0 + per);
  uint32_t local = 0;
  for (int s = s0; s < s1; ++s) local += lens[s];
  uint32_t slab_words;
  uint32_t run = base + block_exclusive_scan(local, warp_tot, slab_words);
  for (int s = s0; s < s1; ++s) {
    offs[s] = 2u * run;
    run += lens[s];
  }
  if (slab != 2 * L - 1) return;

  const uint64_t payload = 2ull * (uint64_t(base) + slab_words);
  const uint64_t total = up16(sec.payload + payload);
  if (tid == 0) {
    offs[n] = uint32_t(payload);  // == offsets[2 L n]
    cg_header hd;
    hd.magic = CG_MAGIC;
    hd.version = p.adjacent ? CG_FORMAT_VERSION_ADJACENT : CG_FORMAT_VERSION;
    hd.level = uint8_t(p.level);
    hd.group = uint8_t(kGroup);
    hd.num_layers = uint32_t(L);
    hd.num_kv_heads = uint32_t(H);
    hd.head_dim = uint32_t(D);
    hd.chunk_tokens = uint32_t(C);
    hd.n_tokens = uint32_t(n);
    hd.prob_bits = kProbBits;
    hd.token_start = uint64_t(t0);
    hd.payload_bytes = payload;
    hd.total_bytes = total;
    hd.reserved = 0;
    const uint4* hs = reinterpret_cast<const uint4*>(&hd);
    for (int i = 0; i < 4; ++i) reinterpret_cast<uint4*>(cont)[i] = hs[i];
    p.out_sizes[chunk] = total;
    if (total > p.out_stride) set_status(p.status, CG_ERR_CAPACITY);
  }
  // Zero the padding after the offsets section and after the payload.
  const uint64_t opad0 = sec.offsets + 4ull * (2ull * L * n + 1);
  if (tid < int(sec.payload - opad0)) cont[opad0 + tid] = 0;
  const uint64_t ppad0 = sec.payload + payload;
  if (total <= p.out_stride && tid < int(total - ppad0)) cont[ppad0 + tid] = 0;
}

__global__ void __launch_bounds__(256) compact_kernel(const EncParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = p.C, L = p.L, H = p.H, D = p.D;
  const uint64_t gs = uint64_t(blockIdx.x) * 8 + warp;
  const uint64_t per_chunk = uint64_t(L) * 2 * C;
  const int chunk = int(gs / per_chunk);
  if (chunk >= p.num_chunks) return;
  const uint64_t rem = gs - uint64_t(chunk) * per_chunk;
  const int slab = int(rem / C), t = int(rem % C);
  const int64_t t0 = p.token_start + int64_t(chunk) * C;
  const int n = int(min(int64_t(C), p.T - t0));
  if (t >= n) return;
  const Sections sec = sections(L, H, D, n);
  uint8_t* cont = p.out + uint64_t(chunk) * p.out_stride;
  const uint32_t o0 = reinterpret_cast<const uint32_t*>(cont + sec.offsets)[uint64_t(slab) * n + t];
  const uint64_t cs = uint64_t(chunk) * L * 2 + slab;
  const uint32_t len = p.lens[cs * C + t];
  if (sec.payload + o0 + 2ull * len > p.out_stride) return;  // capacity error already flagged
  const uint16_t* src =
      reinterpret_cast<const uint16_t*>(p.scratch + (cs * C + t + 1) * scratch_stride(H, D)) - len;
  uint16_t* dst = reinterpret_cast<uint16_t*>(cont + sec.payload + o0);
  // The payload is written in 16-byte aligned chunks; the few u16 words before
  // the first chunk and after the last one are copied one by one.  A chunk's
  // source bytes start at an even offset o within an aligned 16-byte block, so
  // each output word is a funnel shift of two adjacent source words.
  const uint32_t nbytes = 2u * len;
  const uint32_t head = uint32_t((16u - (reinterpret_cast<uintptr_t>(dst) & 15u)) & 15u);
  if (nbytes < head + 16u) {
    for (uint32_t i = lane; i < len; i += 32) dst[i] = src[i];
    return;
  }
  const uint32_t nchunks = (nbytes - head) / 16u;
  const uint32_t tail = (head + nchunks * 16u) / 2u;  // first word after the chunks
  if (lane < head / 2u) dst[lane] = src[lane];
  for (uint32_t i = tail + lane; i < len; i += 32) dst[i] = src[i];
  const uint8_t* sm = reinterpret_cast<const uint8_t*>(src) + head;
  const uint32_t o = uint32_t(reinterpret_cast<uintptr_t>(sm) & 15u);
  const uint4* sa = reinterpret_cast<const uint4*>(sm - o);
  uint4* dm = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(dst) + head);
  const uint32_t q = o >> 2, sh = 8u * (o & 3u);
  for (uint32_t k = lane; k < nchunks; k += 32) {
    const uint4 a = sa[k];
    // the next block holds bytes of this chunk only when o != 0; it then ends
    // at or before the end of the stream's slot
    const uint4 b = o != 0 ? sa[k + 1] : make_uint4(0, 0, 0, 0);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t lo, hi;
      switch (q) {  // warp-uniform
        case 0: lo = w[i]; hi = w[i + 1]; break;
        case 1: lo = w[i + 1]; hi = w[i + 2]; break;
        case 2: lo = w[i + 2]; hi = w[i + 3]; break;
        default: lo = w[i + 3]; hi = w[i + 4]; break;
      }
      r[i] = __funnelshift_r(lo, hi, sh);
    }
    dm[k] = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

// rANS encode, offsets and compaction of one level's symbols (p.sym, p.etab,
// p.slabtot) into its containers (p.out).
cudaError_t launch_streams(const EncParams& p, bool check_f, cudaStream_t stream) {
  cudaError_t err;
  const uint64_t tiles = (p.C + kRThreads - 1) / kRThreads;
  const unsigned rblocks = unsigned(uint64_t(p.num_chunks) * p.L * 2 * tiles);
  if (check_f)
    rans_kernel<true><<<rblocks, kRThreads, 0, stream>>>(p);
  else
    rans_kernel<false><<<rblocks, kRThreads, 0, stream>>>(p);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  offsets_kernel<<<unsigned(uint64_t(p.num_chunks) * p.L * 2), kScanThreads, 0, stream>>>(p);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const uint64_t streams = uint64_t(p.num_chunks) * p.L * 2 * p.C;
  compact_kernel<<<unsigned((streams + 7) / 8), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

namespace {

// Chunks k0, k0 + 1, ... of a call as a call of their own: the containers,
// their sizes, the supplied tables and every workspace section are laid out
// chunk by chunk.
EncParams chunk_tail(const EncParams& p, int k0) {
  EncParams q = p;
  const uint64_t k = uint64_t(k0);
  const uint64_t slabs = uint64_t(p.L) * 2;
  q.token_start = p.token_start + int64_t(k) * p.C;
  q.num_chunks = p.num_chunks - k0;
  const uint64_t sym_per_chunk = slabs * p.H * p.D * p.C;
  const uint64_t etab_per_chunk = slabs * p.H * 256 * 4;
  if (p.out) q.out = p.out + k * p.out_stride;
  if (p.out_sizes) q.out_sizes = p.out_sizes + k;
  if (p.tables_in) q.tables_in = p.tables_in + k * p.tables_stride;
  if (p.sym) q.sym = p.sym + k * sym_per_chunk;
  if (p.etab) q.etab = p.etab + k * etab_per_chunk;
  if (p.slabtot) q.slabtot = p.slabtot + k * slabs;
  q.lens = p.lens + k * slabs * p.C;
  q.scratch = p.scratch + k * slabs * p.C * scratch_stride(p.H, p.D);
  for (int j = 0; j < 3; ++j) {  // the three-level encoder's per-level sections
    if (p.lsym[j]) q.lsym[j] = p.lsym[j] + k * sym_per_chunk;
    if (p.letab[j]) q.letab[j] = p.letab[j] + k * etab_per_chunk;
    if (p.lslabtot[j]) q.lslabtot[j] = p.lslabtot[j] + k * slabs;
    if (p.lout[j]) q.lout[j] = p.lout[j] + k * p.out_stride;
  }
  return q;
}

cudaError_t launch_encode_one(const EncParams& p, int mode, cudaStream_t stream) {
  const QSmem sm = q_smem<1>();
  auto* kern = p.adjacent ? quant_kernel<1, true> : quant_kernel<1, false>;
  const uint64_t qblocks = uint64_t(p.num_chunks) * p.L * 2 * p.H;
  kern<<<unsigned(qblocks), kQThreads, sm.total, stream>>>(p, mode);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess || mode == kModeTablesOnly) return err;
  return launch_streams(p, mode == kModeSuppliedTables, stream);
}

}  // namespace

// A call of two or more chunks runs as two halves, the second on the side
// stream (fork_join): the halves' kernels overlap, which hides most of one
// half's memory-bound compaction and loads behind the other's issue-bound
// rANS encoding.  Without a side stream the call runs on `stream` alone.
cudaError_t launch_encode(const EncParams& p, bool build_only, cudaStream_t stream) {
  const int mode =
      build_only ? kModeTablesOnly : (p.tables_in ? kModeSuppliedTables : kModeEncode);
  const QSmem sm = q_smem<1>();
  auto* kern = p.adjacent ? quant_kernel<1, true> : quant_kernel<1, false>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm.total));
  if (err != cudaSuccess) return err;
  if (!build_only && p.num_chunks >= 2) {
    const int half = (p.num_chunks + 1) / 2;
    EncParams a = p;
    a.num_chunks = half;
    const EncParams b = chunk_tail(p, half);
    bool forked = false;
    err = fork_join(
        stream, [&](cudaStream_t s) { return launch_encode_one(a, mode, s); },
        [&](cudaStream_t s) { return launch_encode_one(b, mode, s); }, &forked);
    if (forked || err != cudaSuccess) return err;
  }
  return launch_encode_one(p, mode, stream);
}

namespace {

// Chunks of a three-level call (p already covers them; k0 is the first one's
// index in the call, whose container sizes are laid out [level][chunk]).
cudaError_t launch_levels_part(const EncParams& p, uint64_t* out_sizes, int total_chunks, int k0,
                               cudaStream_t stream) {
  const QSmem sm = q_smem<3>();
  const uint64_t qblocks = uint64_t(p.num_chunks) * p.L * 2 * p.H;
  quant_kernel<3, false><<<unsigned(qblocks), kQThreads, sm.total, stream>>>(p, kModeEncode);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  for (int j = 0; j < 3; ++j) {
    EncParams q = p;
    q.level = j;
    q.sym = p.lsym[j];
    q.etab = p.letab[j];
    q.slabtot = p.lslabtot[j];
    q.out = p.lout[j];
    q.out_sizes = out_sizes + uint64_t(j) * total_chunks + k0;
    if ((err = launch_streams(q, false, stream)) != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace

// Three levels from one quantiser pass: quant_kernel<3> writes every level's
// symbols, tables and encoder constants; then each level's streams are encoded
// and compacted in turn (the stream lengths and word slots are reused).  As in
// launch_encode, a call of two or more chunks runs as two halves on two
// streams.
cudaError_t launch_encode_levels(const EncParams& p, uint64_t* out_sizes, cudaStream_t stream) {
  const QSmem sm = q_smem<3>();
  cudaError_t err = cudaFuncSetAttribute(quant_kernel<3, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(sm.total));
  if (err != cudaSuccess) return err;
  const int n = p.num_chunks;
  if (n >= 2) {
    const int half = (n + 1) / 2;
    EncParams a = p;
    a.num_chunks = half;
    const EncParams b = chunk_tail(p, half);
    bool forked = false;
    err = fork_join(
        stream, [&](cudaStream_t s) { return launch_levels_part(a, out_sizes, n, 0, s); },
        [&](cudaStream_t s) { return launch_levels_part(b, out_sizes, n, half, s); }, &forked);
    if (forked || err != cudaSuccess) return err;
  }
  return launch_levels_part(p, out_sizes, n, 0, stream);
}

}  // namespace cg
