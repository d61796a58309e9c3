/* synth_cpu.c -- C twin of synth/__init__.py's seeded input generator (same
 * Philox4x32-10 stream and the same fp32 mapping); no MoE arithmetic here. */
#include <stdint.h>
#include <stddef.h>

static inline void philox_round(uint32_t c[4], uint32_t k0, uint32_t k1) {
  uint64_t p0 = (uint64_t)0xD2511F53u * c[0], p1 = (uint64_t)0xCD9E8D57u * c[2];
  uint32_t n0 = (uint32_t)(p1 >> 32) ^ c[1] ^ k0, n2 = (uint32_t)(p0 >> 32) ^ c[3] ^ k1;
  c[0] = n0; c[1] = (uint32_t)p1; c[2] = n2; c[3] = (uint32_t)p0;
}

__attribute__((visibility("default")))
void synth_normal_f32_cpu(float *out, uint64_t n, int count, uint32_t a0, uint32_t a_step,
                          uint32_t b, uint32_t seed, float scale, uint64_t start) {
  for (int m = 0; m < count; ++m)
    for (uint64_t i = 0; i < n; ++i) {
      uint64_t ctr = start + i;
      uint32_t c[4] = {(uint32_t)ctr, (uint32_t)(ctr >> 32), a0 + a_step * (uint32_t)m, b};
      uint32_t k0 = seed, k1 = 0x5EEDC0DEu;
      for (int r = 0; r < 10; ++r) {
        if (r) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
        philox_round(c, k0, k1);
      }
      int32_t s = (int32_t)(c[0] >> 8) + (int32_t)(c[1] >> 8) + (int32_t)(c[2] >> 8) +
                  (int32_t)(c[3] >> 8) - (1 << 25);
      float f = (float)s; /* int -> float rounds to nearest even */
      out[(size_t)m * n + i] = f * scale;
    }
}
