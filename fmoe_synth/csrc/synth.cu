// Device-side filler for the seeded synthetic inputs of the routed-expert MoE
// layer.  Same generator, operation for operation, as fmoe_synth/__init__.py
// (SplitMix64 counter streams, Box-Muller normals with series ln / cos, bf16
// round-to-nearest-even).  Holds none of the layer's arithmetic.
//
// Compiled with -fmad=false: every double step below must be a single IEEE
// operation so that host (numpy) and device produce identical bits.
#include <cstdint>
#include <cstddef>
#include <cmath>
#include <cstring>
#include <cuda_runtime.h>

#define HD __host__ __device__ __forceinline__

namespace {

constexpr uint64_t GAMMA = 0x9E3779B97F4A7C15ull;
constexpr int GROUP = 64;

HD uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

HD uint64_t stream_key(uint64_t seed, uint64_t layer, uint64_t expert, uint64_t tensor) {
  uint64_t key = seed;
  key = mix64(key ^ mix64((layer + 1) * GAMMA));
  key = mix64(key ^ mix64((expert + 1) * GAMMA));
  key = mix64(key ^ mix64((tensor + 1) * GAMMA));
  return key;
}

HD uint64_t draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GAMMA); }

HD double uniform01(uint64_t r) { return (double)((r >> 11) + 1) * 0x1p-53; }

// ln(u), u in (0,1]: u = m 2^e, m in [sqrt(1/2), sqrt(2)), ln m = 2 atanh((m-1)/(m+1)).
HD double ln_unit(double u) {
  int e;
  double m = frexp(u, &e);
  if (m < 0.7071067811865476) { m = m * 2.0; e = e - 1; }
  double t = (m - 1.0) / (m + 1.0);
  double t2 = t * t;
  double s = 1.0 / 23.0;
  s = (1.0 / 21.0) + t2 * s;
  s = (1.0 / 19.0) + t2 * s;
  s = (1.0 / 17.0) + t2 * s;
  s = (1.0 / 15.0) + t2 * s;
  s = (1.0 / 13.0) + t2 * s;
  s = (1.0 / 11.0) + t2 * s;
  s = (1.0 / 9.0) + t2 * s;
  s = (1.0 / 7.0) + t2 * s;
  s = (1.0 / 5.0) + t2 * s;
  s = (1.0 / 3.0) + t2 * s;
  s = t2 * s;
  double tt = 2.0 * t;
  double lnm = tt + tt * s;
  return (double)e * 0.6931471805599453 + lnm;
}

// cos(2 pi u), u in (0,1]: exact reflections to [0, 1/8], Taylor series of cos / sin.
HD double cos_2pi(double u) {
  double v = (u < 0.5) ? u : (u - 1.0);
  double a = fabs(v);
  bool neg = a > 0.25;
  if (neg) a = 0.5 - a;
  bool use_sin = a > 0.125;
  double b = use_sin ? (0.25 - a) : a;
  double th = 6.283185307179586 * b;
  double th2 = th * th;
  double r;
  if (!use_sin) {
    double c = -(1.0 / 6402373705728000.0);            // -1/18!
    c = (1.0 / 20922789888000.0) + th2 * c;             //  1/16!
    c = -(1.0 / 87178291200.0) + th2 * c;               // -1/14!
    c = (1.0 / 479001600.0) + th2 * c;                  //  1/12!
    c = -(1.0 / 3628800.0) + th2 * c;                   // -1/10!
    c = (1.0 / 40320.0) + th2 * c;                      //  1/8!
    c = -(1.0 / 720.0) + th2 * c;                       // -1/6!
    c = (1.0 / 24.0) + th2 * c;                         //  1/4!
    c = -(1.0 / 2.0) + th2 * c;                         // -1/2!
    c = 1.0 + th2 * c;
    r = c;
  } else {
    double s = -(1.0 / 121645100408832000.0);          // -1/19!
    s = (1.0 / 355687428096000.0) + th2 * s;            //  1/17!
    s = -(1.0 / 1307674368000.0) + th2 * s;             // -1/15!
    s = (1.0 / 6227020800.0) + th2 * s;                 //  1/13!
    s = -(1.0 / 39916800.0) + th2 * s;                  // -1/11!
    s = (1.0 / 362880.0) + th2 * s;                     //  1/9!
    s = -(1.0 / 5040.0) + th2 * s;                      // -1/7!
    s = (1.0 / 120.0) + th2 * s;                        //  1/5!
    s = -(1.0 / 6.0) + th2 * s;                         // -1/3!
    s = 1.0 + th2 * s;
    r = th * s;
  }
  return neg ? -r : r;
}

HD double normal_at(uint64_t key, uint64_t j) {
  double u1 = uniform01(draw(key, 2 * j));
  double u2 = uniform01(draw(key, 2 * j + 1));
  return sqrt(-2.0 * ln_unit(u1)) * cos_2pi(u2);
}

HD uint16_t bf16_bits(double v) {
  if (v == 0.0) return signbit(v) ? (uint16_t)0x8000 : (uint16_t)0;
  int e;
  double m = frexp(v, &e);
  double q = rint(m * 256.0);
  double r = ldexp(q, e - 8);
  float f = (float)r;
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

HD double bf16_value(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

HD uint32_t q_word(uint64_t key, uint64_t i) {
  uint64_t r = draw(key, i >> 1);
  return (i & 1) ? (uint32_t)(r >> 32) : (uint32_t)r;
}

HD uint32_t sb_pair(uint64_t key, uint64_t j, double center) {
  double ns = normal_at(key, 2 * j);
  double nb = normal_at(key, 2 * j + 1);
  uint16_t s = bf16_bits(fabs(ns) * 0.02);
  uint16_t b = bf16_bits(-center * bf16_value(s) + 1e-3 * nb);
  return (uint32_t)s | ((uint32_t)b << 16);
}

HD size_t al256(size_t n) { return (n + 255) / 256 * 256; }

struct Layout {
  size_t qh, qi, sh, si, o_gu_sb, o_d_q, o_d_sb, size;
  HD Layout(int H, int I, int bits) {
    qh = (size_t)H * bits / 8;
    qi = (size_t)I * bits / 8;
    sh = (size_t)(H / GROUP) * 4;
    si = (size_t)(I / GROUP) * 4;
    o_gu_sb = al256((size_t)I * 2 * qh);
    o_d_q = al256(o_gu_sb + (size_t)I * 2 * sh);
    o_d_sb = al256(o_d_q + (size_t)H * qi);
    size = al256(o_d_sb + (size_t)H * si);
  }
};

enum { T_GATE_Q = 0, T_UP_Q, T_DOWN_Q, T_GATE_SB, T_UP_SB, T_DOWN_SB, T_ROUTER, T_SHARED_GATE,
       T_ROUTER_BIAS, T_X };

// One thread per 32-bit word of the record (padding words written as zero).
__global__ void k_fill_records(uint8_t* base, int H, int I, int bits, uint64_t seed, int layer,
                               int expert0, int n_experts) {
  Layout L(H, I, bits);
  const size_t words_per_rec = L.size / 4;
  const size_t total = words_per_rec * (size_t)n_experts;
  const double center = bits == 4 ? 8.0 : 2.0;
  const size_t wh = (size_t)H * bits / 32, wi = (size_t)I * bits / 32;
  const size_t gh = H / GROUP, gi = I / GROUP;
  for (size_t g = blockIdx.x * (size_t)blockDim.x + threadIdx.x; g < total;
       g += (size_t)gridDim.x * blockDim.x) {
    const int e = expert0 + (int)(g / words_per_rec);
    const size_t off = (g % words_per_rec) * 4;
    uint32_t v = 0;
    if (off < (size_t)I * 2 * L.qh) {
      size_t w = off / 4, r = w / (2 * wh), rem = w % (2 * wh);
      int t = rem < wh ? T_GATE_Q : T_UP_Q;
      size_t c = rem % wh;
      v = q_word(stream_key(seed, layer, e, t), r * wh + c);
    } else if (off >= L.o_gu_sb && off < L.o_gu_sb + (size_t)I * 2 * L.sh) {
      size_t w = (off - L.o_gu_sb) / 4, r = w / (2 * gh), rem = w % (2 * gh);
      int t = rem < gh ? T_GATE_SB : T_UP_SB;
      size_t c = rem % gh;
      v = sb_pair(stream_key(seed, layer, e, t), r * gh + c, center);
    } else if (off >= L.o_d_q && off < L.o_d_q + (size_t)H * L.qi) {
      size_t w = (off - L.o_d_q) / 4;
      v = q_word(stream_key(seed, layer, e, T_DOWN_Q), w);
    } else if (off >= L.o_d_sb && off < L.o_d_sb + (size_t)H * L.si) {
      size_t w = (off - L.o_d_sb) / 4;
      v = sb_pair(stream_key(seed, layer, e, T_DOWN_SB), w, center);
    }
    reinterpret_cast<uint32_t*>(base)[g] = v;
  }
  (void)wi; (void)gi;
}

__global__ void k_fill_normals_f32(float* dst, size_t n, uint64_t key, double scale) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = (float)(scale * normal_at(key, i));
}

// One thread per token: left-to-right sum of squares, as the host generator.
__global__ void k_fill_x(uint16_t* dst, uint64_t seed, int t0, int T, int H) {
  int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  uint64_t key = stream_key(seed, 0, (uint64_t)(t0 + t), T_X);
  double ss = 0.0;
  for (int c = 0; c < H; ++c) { double z = normal_at(key, c); ss = ss + z * z; }
  double r = sqrt(ss / (double)H + 1e-6);
  for (int c = 0; c < H; ++c) dst[(size_t)t * H + c] = bf16_bits(normal_at(key, c) / r);
}

int grid_for(size_t n) {
  size_t g = (n + 255) / 256;
  return (int)(g > 148 * 64 ? 148 * 64 : (g == 0 ? 1 : g));
}

}  // namespace

extern "C" {

size_t fmoe_synth_record_bytes(int H, int I, int bits) { return Layout(H, I, bits).size; }

// Fill n_experts consecutive records (experts expert0 .. expert0+n-1 of one layer).
int fmoe_synth_fill_records(void* dst, int H, int I, int bits, uint64_t seed, int layer,
                            int expert0, int n_experts, cudaStream_t stream) {
  size_t words = Layout(H, I, bits).size / 4 * (size_t)n_experts;
  k_fill_records<<<grid_for(words), 256, 0, stream>>>((uint8_t*)dst, H, I, bits, seed, layer,
                                                      expert0, n_experts);
  return (int)cudaGetLastError();
}

int fmoe_synth_fill_router(float* dst, uint64_t seed, int layer, int E, int H, cudaStream_t s) {
  size_t n = (size_t)E * H;
  k_fill_normals_f32<<<grid_for(n), 256, 0, s>>>(dst, n, stream_key(seed, layer, 0, T_ROUTER), 0.02);
  return (int)cudaGetLastError();
}

int fmoe_synth_fill_shared_gate(float* dst, uint64_t seed, int layer, int H, cudaStream_t s) {
  k_fill_normals_f32<<<grid_for(H), 256, 0, s>>>(dst, H, stream_key(seed, layer, 0, T_SHARED_GATE), 0.02);
  return (int)cudaGetLastError();
}

int fmoe_synth_fill_router_bias(float* dst, uint64_t seed, int layer, int E, cudaStream_t s) {
  k_fill_normals_f32<<<grid_for(E), 256, 0, s>>>(dst, E, stream_key(seed, layer, 0, T_ROUTER_BIAS), 1.0);
  return (int)cudaGetLastError();
}

int fmoe_synth_fill_x(uint16_t* dst, uint64_t seed, int t0, int T, int H, cudaStream_t s) {
  k_fill_x<<<(T + 127) / 128, 128, 0, s>>>(dst, seed, t0, T, H);
  return (int)cudaGetLastError();
}

// Host execution of the same generator code (for CPU cross-checks against numpy).
void fmoe_synth_host_normals(double* out, uint64_t key, uint64_t start, uint64_t n) {
  for (uint64_t i = 0; i < n; ++i) out[i] = normal_at(key, start + i);
}

void fmoe_synth_host_record(uint8_t* dst, int H, int I, int bits, uint64_t seed, int layer, int expert) {
  Layout L(H, I, bits);
  const double center = bits == 4 ? 8.0 : 2.0;
  const size_t wh = (size_t)H * bits / 32;
  const size_t gh = H / GROUP;
  uint32_t* w32 = reinterpret_cast<uint32_t*>(dst);
  for (size_t g = 0; g < L.size / 4; ++g) {
    size_t off = g * 4;
    uint32_t v = 0;
    if (off < (size_t)I * 2 * L.qh) {
      size_t w = off / 4, r = w / (2 * wh), rem = w % (2 * wh);
      v = q_word(stream_key(seed, layer, expert, rem < wh ? T_GATE_Q : T_UP_Q), r * wh + rem % wh);
    } else if (off >= L.o_gu_sb && off < L.o_gu_sb + (size_t)I * 2 * L.sh) {
      size_t w = (off - L.o_gu_sb) / 4, r = w / (2 * gh), rem = w % (2 * gh);
      v = sb_pair(stream_key(seed, layer, expert, rem < gh ? T_GATE_SB : T_UP_SB), r * gh + rem % gh, center);
    } else if (off >= L.o_d_q && off < L.o_d_q + (size_t)H * L.qi) {
      v = q_word(stream_key(seed, layer, expert, T_DOWN_Q), (off - L.o_d_q) / 4);
    } else if (off >= L.o_d_sb && off < L.o_d_sb + (size_t)H * L.si) {
      v = sb_pair(stream_key(seed, layer, expert, T_DOWN_SB), (off - L.o_d_sb) / 4, center);
    }
    w32[g] = v;
  }
}

}  // extern "C"
