// kvsynth.cu -- seeded synthetic fp16 KV caches (input generator only; none of
// the codec's arithmetic lives here).
//
// Definition (identical to the numpy twin in synth/__init__.py):
//   key      = (seed mod 2^32, seed div 2^32)
//   channel  ch = ((l*2 + kv)*H + h)*D + d
//   Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
//   easy as 1, 2, 3", SC'11) with counter (ch, k, 0, tag):
//     tag 1, k = 0 : channel draw  r -> amplitude exp(0.5 z) * (u3 < p ? m : 1)
//     tag 2, k     : the normals of tokens 2k and 2k+1
//   uniforms u1 = (r0 + 1) 2^-32 in (0, 1], u2 = r1 2^-32, u3 = r2 2^-32;
//   Box-Muller: rad = sqrt(-2 ln u1), z0 = rad cos(2 pi u2), z1 = rad sin(2 pi u2)
//   AR(1) walk along the whole sequence: x_0 = e_0, x_t = rho x_{t-1} + sigma e_t,
//   sigma = sqrt(1 - rho^2); value = fp16_rn(amplitude * x_t), all in fp64.
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

__device__ __forceinline__ void box_muller(uint32_t a, uint32_t b, double& z0, double& z1) {
  const double u1 = (double(a) + 1.0) * 2.3283064365386963e-10;  // 2^-32
  const double u2 = double(b) * 2.3283064365386963e-10;
  const double rad = sqrt(__dmul_rn(-2.0, log(u1)));
  const double th = __dmul_rn(6.283185307179586, u2);
  z0 = __dmul_rn(rad, cos(th));
  z1 = __dmul_rn(rad, sin(th));
}

__global__ void gen_kernel(uint16_t* out, int L, int H, int D, int64_t T, uint32_t k0,
                           uint32_t k1, double rho, double p_out, double m_out) {
  const int64_t chans = int64_t(L) * 2 * H * D;
  const int64_t ch = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (ch >= chans) return;
  const int64_t hd = int64_t(H) * D;
  const int64_t slab = ch / hd, inrow = ch % hd;
  uint16_t* col = out + slab * T * hd + inrow;

  const uint4 cr = philox4x32_10(make_uint4(uint32_t(ch), 0u, 0u, 1u), k0, k1);
  double z, unused;
  box_muller(cr.x, cr.y, z, unused);
  const double u3 = double(cr.z) * 2.3283064365386963e-10;
  const double amp = __dmul_rn(exp(__dmul_rn(0.5, z)), u3 < p_out ? m_out : 1.0);
  const double sigma = sqrt(__dadd_rn(1.0, -__dmul_rn(rho, rho)));

  double x = 0.0;
  for (int64_t t = 0; t < T; t += 2) {
    const uint4 r = philox4x32_10(make_uint4(uint32_t(ch), uint32_t(t >> 1), 0u, 2u), k0, k1);
    double e0, e1;
    box_muller(r.x, r.y, e0, e1);
    x = t == 0 ? e0 : __dadd_rn(__dmul_rn(rho, x), __dmul_rn(sigma, e0));
    col[t * hd] = __half_as_ushort(__double2half(__dmul_rn(amp, x)));
    if (t + 1 < T) {
      x = __dadd_rn(__dmul_rn(rho, x), __dmul_rn(sigma, e1));
      col[(t + 1) * hd] = __half_as_ushort(__double2half(__dmul_rn(amp, x)));
    }
  }
}

}  // namespace

extern "C" int kvsynth_generate(uint16_t* out_dev, int L, int H, int D, int64_t T,
                                uint64_t seed, double rho, double p_out, double m_out,
                                cudaStream_t stream) {
  if (out_dev == nullptr || L < 1 || H < 1 || D < 1 || T < 1) return 1;
  const int64_t chans = int64_t(L) * 2 * H * D;
  const int threads = 128;
  const int64_t blocks = (chans + threads - 1) / threads;
  gen_kernel<<<unsigned(blocks), threads, 0, stream>>>(out_dev, L, H, D, T,
                                                       uint32_t(seed & 0xFFFFFFFFu),
                                                       uint32_t(seed >> 32), rho, p_out, m_out);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
