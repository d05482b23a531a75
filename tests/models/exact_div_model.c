/* A host model of the quantizers' division-free quotient (CPU, no GPU).
 *
 * Every quotient of the NVFP4 recipe is x / d with d fixed for a tensor
 * (d = RN(6 s_t)) or a block (d = RN(s_b s_t)).  The kernels hold, per d,
 * y_rn = RN(1/d), y_rd = RD(1/d) and y_lo = RN((1 - d y_rd) y_rd), negated, and
 * compute q0 = RN(x y_rd + RN(x y_lo)) followed by one remainder correction
 * q = RN(q0 + (x - d q0) y_rn) (Markstein's theorem), all on the negated
 * dividend -x.  This model restates those steps with C99 fmaf (one rounding
 * per operation) and compares q with the IEEE quotient x / d bit for bit.
 *
 * Output: one line per case, "<name> <checks> <mismatches>".  A quotient below
 * 2^-10 codes to zero in E2M1 and E4M3 whatever its last bits, so for those
 * only the sign is compared.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float bits2f(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t f2bits(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

typedef struct { float d, ny_rd, ny_lo, ny_rn; } Ent;

static Ent entry(float d) {
  Ent e;
  float y_rn = 1.0f / d, y_rd = y_rn;
  if (fmaf(-d, y_rn, 1.0f) < 0.0f) y_rd = nextafterf(y_rn, 0.0f); /* RD(1/d) */
  float rho = fmaf(-d, y_rd, 1.0f);
  e.d = d;
  e.ny_rd = -y_rd;
  e.ny_lo = -(rho * y_rd);
  e.ny_rn = -y_rn;
  return e;
}

static float quot(const Ent* e, float x) {
  float nx = -x;
  float q0 = fmaf(nx, e->ny_rd, nx * e->ny_lo);
  float r = fmaf(e->d, q0, nx);
  return fmaf(r, e->ny_rn, q0);
}

static int agree(float q, float ref) {
  if (fabsf(ref) < 0x1p-10f) return signbit(q) == signbit(ref) && fabsf(q) < 0x1p-9f;
  return f2bits(q) == f2bits(ref);
}

int main(int argc, char** argv) {
  unsigned d_stride = 1u << 7; /* divisor significands: every 128th of 2^23 */
  if (argc > 1) sscanf(argv[1], "%u", &d_stride);
  /* 1. every positive and negative normal bf16 dividend with x / d in [2^-7, 2^5) */
  long long n = 0, bad = 0;
  for (uint32_t m = 0; m < (1u << 23); m += d_stride) {
    float d = bits2f(0x3F800000u | m);
    Ent e = entry(d);
    for (int ex = -6; ex <= 4; ++ex)
      for (uint32_t xm = 0; xm < 128; ++xm)
        for (uint32_t s = 0; s < 2; ++s) {
          float x = bits2f((s << 31) | ((uint32_t)(127 + ex) << 23) | (xm << 16));
          ++n;
          bad += !agree(quot(&e, x), x / d);
        }
  }
  printf("bf16_dividends %lld %lld\n", n, bad);
  /* 2. random binary32 dividends and divisors (xorshift64) */
  uint64_t st = 0x243F6A8885A308D3ull;
  n = bad = 0;
  for (long i = 0; i < 4000000; ++i) {
    st ^= st << 13; st ^= st >> 7; st ^= st << 17;
    float d = bits2f(0x3F800000u | (uint32_t)(st & 0x7FFFFF));
    int ex = (int)((st >> 46) % 12) - 7;
    float x = bits2f((uint32_t)((st >> 60) & 1) << 31 | ((uint32_t)(127 + ex) << 23) |
                     (uint32_t)((st >> 23) & 0x7FFFFF));
    Ent e = entry(d);
    ++n;
    bad += !agree(quot(&e, x), x / d);
  }
  printf("binary32_dividends %lld %lld\n", n, bad);
  /* 3. exact quotients: x = b d for every E2M1 boundary b and E4M3-like d */
  static const float b[] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f, 6.0f, 448.0f};
  n = bad = 0;
  for (uint32_t m = 0; m < 8; ++m)
    for (int ex = -9; ex <= 8; ++ex)
      for (int t = -3; t <= 3; ++t) {
        float d = ldexpf(1.0f + m / 8.0f, ex) * ldexpf(1.0f, t * 11); /* s_b s_t */
        Ent e = entry(d);
        for (int i = 0; i < 9; ++i) {
          float x = b[i] * d;
          if (x != (double)b[i] * d) continue;
          ++n;
          bad += !agree(quot(&e, x), x / d);
          ++n;
          bad += !agree(quot(&e, -x), -x / d);
        }
      }
  printf("exact_ties %lld %lld\n", n, bad);
  /* 4. every bf16 dividend (zeros and subnormals included) over the divisor
   * range the recipe's domain allows, d in [2^-117, 2^109] */
  static const float ds[] = {0x1p-117f, 0x1.8p-100f, 0x1.234566p-60f, 1.0f,
                             0x1.fffffep0f, 0x1.5p20f, 0x1.ffp100f, 0x1p109f};
  n = bad = 0;
  for (int i = 0; i < 8; ++i) {
    Ent e = entry(ds[i]);
    for (uint32_t xb = 0; xb < 0x10000u; ++xb) {
      float x = bits2f(xb << 16);
      if (!isfinite(x)) continue;
      float ref = x / ds[i];
      if (fabsf(ref) > 8.0f) continue; /* block quotients stay below 6.4 */
      ++n;
      bad += !agree(quot(&e, x), ref);
    }
  }
  printf("edge_dividends %lld %lld\n", n, bad);
  return 0;
}
