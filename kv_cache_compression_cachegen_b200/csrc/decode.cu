// decode.cu -- fused rANS decode -> dequantise -> fp16 store (cg_decode and
// cg_decode_into).
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
//                  all threads build the slot table of head it + 1.
// The anchor warp runs one head ahead so that the reconstructed anchors a_g of
// head it-1 (fp32, in shared memory) are ready when the delta warps need them;
// one __syncthreads per head separates the iterations.
//
// Per symbol a thread does one shared-memory slot lookup, the rANS state
// update, an optional 16-bit refill from its own stream (L1-cached global
// loads), and the dequantisation a + (float)q * s with IEEE round-to-nearest
// adds and multiplies (no contraction).  (float)q * step is exact-rounded once,
// so it is read from a 255-entry table of the layer's products.
#include <cuda_fp16.h>

#include "cg_common.cuh"

namespace cg {
namespace {

constexpr int kUnitGroups = 32;
constexpr int kDeltaPerGroup = kGroup - 1;             // 9
constexpr int kWarps = 1 + kDeltaPerGroup;             // anchor warp + 9 delta warps
constexpr int kThreads = 32 * kWarps;                  // 320
constexpr int kUnitTokens = kUnitGroups * kGroup;      // 320
constexpr int kCumStride = 258;                        // u16 per head: cum[0..256] + pad

// Dynamic shared memory layout (byte offsets), a function of H and D.
struct DecSmem {
  uint32_t tbl;     // u32 [3][4096]   slot tables, packed (f << 20) | (u << 12) | (slot - cum)
  uint32_t ahat;    // f32 [2][32][D + 4]  reconstructed anchors of the last two heads
  uint32_t cum;     // u16 [H][258]    cumulative frequencies of every head
  uint32_t lut;     // f32 [256]       (float)(u - 127) * step for this layer
  uint32_t single;  // i32 [H]         symbol of a one-symbol table, else -1
  uint32_t total;
};

__host__ __device__ inline uint32_t al16(uint32_t v) { return (v + 15u) & ~15u; }

__host__ __device__ inline DecSmem dec_smem(int H, int D) {
  DecSmem s;
  s.tbl = 0;
  s.ahat = al16(s.tbl + 3u * 4096u * 4u);
  s.cum = al16(s.ahat + 2u * kUnitGroups * uint32_t(D + 4) * 4u);
  s.lut = al16(s.cum + uint32_t(H) * kCumStride * 2u);
  s.single = al16(s.lut + 256u * 4u);
  s.total = al16(s.single + uint32_t(H) * 4u);
  return s;
}

__device__ __forceinline__ uint16_t ldg_u16(const uint16_t* p) { return __ldg(p); }

// Fill the 4096-entry slot table of one head: thread tid covers slots
// [tid*4096/kThreads, (tid+1)*4096/kThreads).  The symbol of the first slot is
// found by binary search over the cumulative frequencies; the rest by walking.
__device__ __forceinline__ void fill_table(uint32_t* tbl, const uint16_t* cum, int tid) {
  const int s0 = (tid * int(kM)) / kThreads;
  const int s1 = ((tid + 1) * int(kM)) / kThreads;
  int lo = 0, hi = kAlphabet;  // cum[lo] <= s0 < cum[hi]; cum[255] == 4096
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (int(cum[mid]) <= s0) lo = mid; else hi = mid;
  }
  int u = lo;
  int cc = cum[u], cn = cum[u + 1];
  for (int s = s0; s < s1; ++s) {
    while (cn <= s) {
      ++u;
      cc = cn;
      cn = cum[u + 1];
    }
    tbl[s] = (uint32_t(cn - cc) << 20) | (uint32_t(u) << 12) | uint32_t(s - cc);
  }
}

// One rANS decode step: returns the packed table entry of the decoded symbol.
template <bool kClamp>
__device__ __forceinline__ uint32_t rans_step(uint32_t& x, uint64_t& p, uint32_t& w,
                                              const uint32_t* __restrict__ tbl,
                                              const uint16_t* __restrict__ w16, uint64_t limit) {
  const uint32_t e = tbl[x & (kM - 1)];
  x = (e >> 20) * (x >> kProbBits) + (e & (kM - 1));
  if (x < kRansL) {
    x = (x << 16) | w;
    ++p;
    const uint64_t q = kClamp ? (p < limit ? p : limit - 1) : p;
    w = ldg_u16(w16 + q);
  }
  return e;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Delta lane: decode head h of its stream into 8-value blocks.
template <bool kClamp>
__device__ __forceinline__ void decode_delta_head(uint32_t& x, uint64_t& p, uint32_t& w,
                                                  const uint32_t* __restrict__ tbl,
                                                  const float* __restrict__ lut,
                                                  const float* __restrict__ arow,
                                                  uint16_t* __restrict__ orow, int D,
                                                  const uint16_t* __restrict__ w16,
                                                  uint64_t limit) {
  for (int d0 = 0; d0 < D; d0 += 8) {
    const float4 a0 = *reinterpret_cast<const float4*>(arow + d0);
    const float4 a1 = *reinterpret_cast<const float4*>(arow + d0 + 4);
    const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    uint32_t hv[4];
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const uint32_t e0 = rans_step<kClamp>(x, p, w, tbl, w16, limit);
      const float v0 = __fadd_rn(a[k], lut[(e0 >> 12) & 0xFF]);
      const uint32_t e1 = rans_step<kClamp>(x, p, w, tbl, w16, limit);
      const float v1 = __fadd_rn(a[k + 1], lut[(e1 >> 12) & 0xFF]);
      hv[k >> 1] = pack_half2(v0, v1);
    }
    *reinterpret_cast<uint4*>(orow + d0) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
  }
}

// Anchor lane: decode head h, write fp16(a) and keep a (fp32) for the deltas.
template <bool kClamp>
__device__ __forceinline__ void decode_anchor_head(uint32_t& x, uint64_t& p, uint32_t& w,
                                                   const uint32_t* __restrict__ tbl,
                                                   const float* __restrict__ zp,
                                                   const float* __restrict__ sc,
                                                   float* __restrict__ arow,
                                                   uint16_t* __restrict__ orow, int D,
                                                   const uint16_t* __restrict__ w16,
                                                   uint64_t limit) {
  for (int d0 = 0; d0 < D; d0 += 8) {
    const float4 z0 = __ldg(reinterpret_cast<const float4*>(zp + d0));
    const float4 z1 = __ldg(reinterpret_cast<const float4*>(zp + d0 + 4));
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(sc + d0));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(sc + d0 + 4));
    const float z[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
    const float s[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t e = rans_step<kClamp>(x, p, w, tbl, w16, limit);
      const int c = int((e >> 12) & 0xFF) - 127;
      v[k] = __fadd_rn(z[k], __fmul_rn(float(c), s[k]));
    }
    *reinterpret_cast<float4*>(arow + d0) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(arow + d0 + 4) = make_float4(v[4], v[5], v[6], v[7]);
    *reinterpret_cast<uint4*>(orow + d0) =
        make_uint4(pack_half2(v[0], v[1]), pack_half2(v[2], v[3]), pack_half2(v[4], v[5]),
                   pack_half2(v[6], v[7]));
  }
}

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
    // Header validation (every CTA of the chunk checks the same 64 bytes).
    const uint4* hp = reinterpret_cast<const uint4*>(base);
    cg_header h;
    uint4* hd = reinterpret_cast<uint4*>(&h);
    for (int i = 0; i < 4; ++i) hd[i] = __ldg(hp + i);
    int err = 0;
    if (h.magic != CG_MAGIC || h.version != CG_FORMAT_VERSION || h.group != kGroup ||
        h.prob_bits != kProbBits || h.reserved != 0)
      err = CG_ERR_CORRUPT;
    else if (h.level != uint32_t(p.level) || h.num_layers != uint32_t(L) ||
             h.num_kv_heads != uint32_t(H) || h.head_dim != uint32_t(D) ||
             h.chunk_tokens != uint32_t(p.C))
      err = CG_ERR_MISMATCH;
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
  uint16_t* cum = reinterpret_cast<uint16_t*>(smem + sm.cum);
  float* lut = reinterpret_cast<float*>(smem + sm.lut);
  int* single = reinterpret_cast<int*>(smem + sm.single);
  const int astride = D + 4;
  const int warp = tid >> 5, lane = tid & 31;
  const int slab = l * 2 + kv;

  // Cumulative frequencies of every head of this (l, kv): warp-wide scans.
  const uint16_t* freq = reinterpret_cast<const uint16_t*>(base + sec.freq) + size_t(slab) * H * 256;
  for (int h = warp; h < H; h += kWarps) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(freq + h * 256) + lane);
    const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = wv[i] & 0xFFFF;
      f[2 * i + 1] = wv[i] >> 16;
    }
    uint32_t local = 0;
    int one = -1;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      local += f[i];
      if (f[i] == kM) one = lane * 8 + i;
      if (f[i] > kM) bad = true;
    }
    if (lane == 31 && f[7] != 0) bad = true;  // symbol 255 never exists
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    uint32_t run = incl - local;
    uint16_t* ch = cum + h * kCumStride;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      ch[lane * 8 + i] = uint16_t(run < kM ? run : kM);
      run += f[i];
    }
    if (lane == 31) ch[256] = uint16_t(kM);
    one = __reduce_max_sync(0xFFFFFFFFu, one);
    if (lane == 0) single[h] = one;
    if (__any_sync(0xFFFFFFFFu, bad) || total != kM) {
      if (lane == 0) s_bad = 1;
    }
  }
  const float step = step_of(p.level, l, L);
  for (int u = tid; u < 256; u += kThreads) lut[u] = __fmul_rn(float(u - 127), step);
  __syncthreads();
  if (s_bad) {
    if (tid == 0) set_status(p.status, CG_ERR_CORRUPT);
    return;
  }
  fill_table(tbl, cum, tid);

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
  const uint16_t* w16 = reinterpret_cast<const uint16_t*>(base);
  const uint64_t limit = s_total / 2;  // u16 words readable in this container
  const uint32_t* offs = reinterpret_cast<const uint32_t*>(base + sec.offsets);
  uint64_t pw = 0, pend = 0;
  uint32_t x = kRansL, w = 0;
  if (active) {
    const uint64_t s = uint64_t(slab) * n + token;
    const uint32_t o0 = __ldg(offs + s), o1 = __ldg(offs + s + 1);
    const uint64_t payload = s_total - sec.payload;  // includes the final padding
    if (o1 < o0 || uint64_t(o1) > payload || ((o1 - o0) & 1u) || o1 - o0 < 4) {
      set_status(p.status, CG_ERR_CORRUPT);
      active = false;
    } else {
      pw = (sec.payload + o0) / 2;
      pend = (sec.payload + o1) / 2;
      x = (uint32_t(ldg_u16(w16 + pw)) << 16) | ldg_u16(w16 + pw + 1);
      pw += 2;
      w = pw < limit ? ldg_u16(w16 + pw) : 0;
      if (x < kRansL) {
        set_status(p.status, CG_ERR_CORRUPT);
        active = false;
      }
    }
  }
  uint16_t* orow;
  if (p.into)
    orow = p.out + ((uint64_t(slab) * p.total_tokens + uint64_t(s_tstart) + token) * H) * D;
  else
    orow = p.out + uint64_t(chunk) * (uint64_t(L) * 2 * p.C * H * D) +
           ((uint64_t(slab) * n + token) * H) * D;
  const float* zp_sec = reinterpret_cast<const float*>(base + sec.zp) + size_t(slab) * H * D;
  const float* sc_sec = reinterpret_cast<const float*>(base + sec.scale) + size_t(slab) * H * D;
  __syncthreads();

  for (int it = 0; it <= H; ++it) {
    if (it + 1 < H) fill_table(tbl + ((it + 1) % 3) * kM, cum + (it + 1) * kCumStride, tid);
    if (warp == 0) {
      if (it < H && active) {
        const int h = it;
        const uint32_t* tb = tbl + (h % 3) * kM;
        float* arow = ahat + ((h & 1) * kUnitGroups + g_local) * astride;
        const int one = single[h];
        if (one >= 0) {
          const float c = float(one - 127);
          for (int d0 = 0; d0 < D; d0 += 8) {
            float v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
              v[k] = __fadd_rn(zp_sec[h * D + d0 + k], __fmul_rn(c, sc_sec[h * D + d0 + k]));
#pragma unroll
            for (int k = 0; k < 8; ++k) arow[d0 + k] = v[k];
            *reinterpret_cast<uint4*>(orow + h * D + d0) =
                make_uint4(pack_half2(v[0], v[1]), pack_half2(v[2], v[3]),
                           pack_half2(v[4], v[5]), pack_half2(v[6], v[7]));
          }
        } else if (pw + uint64_t(D) + 1 <= limit) {
          decode_anchor_head<false>(x, pw, w, tb, zp_sec + h * D, sc_sec + h * D, arow,
                                    orow + h * D, D, w16, limit);
        } else {
          decode_anchor_head<true>(x, pw, w, tb, zp_sec + h * D, sc_sec + h * D, arow,
                                   orow + h * D, D, w16, limit);
        }
      }
    } else if (it >= 1 && active) {
      const int h = it - 1;
      const uint32_t* tb = tbl + (h % 3) * kM;
      const float* arow = ahat + ((h & 1) * kUnitGroups + g_local) * astride;
      const int one = single[h];
      if (one >= 0) {
        const float v = lut[one];
        for (int d0 = 0; d0 < D; d0 += 8) {
          uint32_t hv[4];
#pragma unroll
          for (int k = 0; k < 8; k += 2)
            hv[k >> 1] = pack_half2(__fadd_rn(arow[d0 + k], v), __fadd_rn(arow[d0 + k + 1], v));
          *reinterpret_cast<uint4*>(orow + h * D + d0) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        }
      } else if (pw + uint64_t(D) + 1 <= limit) {
        decode_delta_head<false>(x, pw, w, tb, lut, arow, orow + h * D, D, w16, limit);
      } else {
        decode_delta_head<true>(x, pw, w, tb, lut, arow, orow + h * D, D, w16, limit);
      }
    }
    __syncthreads();
  }
  if (active && (x != kRansL || pw != pend)) set_status(p.status, CG_ERR_CORRUPT);
}

}  // namespace

cudaError_t launch_decode(const DecParams& p, cudaStream_t stream) {
  const DecSmem sm = dec_smem(p.H, p.D);
  static thread_local int configured_bytes = -1;
  cudaError_t err = cudaSuccess;
  if (configured_bytes < int(sm.total)) {
    err = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(sm.total));
    if (err != cudaSuccess) return err;
    configured_bytes = int(sm.total);
  }
  const uint64_t blocks = uint64_t(p.num_chunks) * p.L * 2 * p.units_per_slab;
  decode_kernel<<<unsigned(blocks), kThreads, sm.total, stream>>>(p);
  return cudaGetLastError();
}

int decode_units_per_slab(int C) {
  const int groups = (C + kGroup - 1) / kGroup;
  return (groups + kUnitGroups - 1) / kUnitGroups;
}

}  // namespace cg
