/* Brute force over all 3^16 two-bit code patterns of a 4x4 head (test of the CPU oracle).
 * For each trial: random fp16 row scales, column scales {1, x, y, z} in a random column order.
 * A pattern is "valid" (one that quantize can produce) when every row holds a +-1 in a column
 * of scale 1 and every column holds a +-1; valid patterns must survive
 * quantize(dequantize(P)) byte for byte. For a sample of the other patterns, P' = Q(D(P))
 * must itself survive. Prints: valid=N mismatch=N unstable=N checked_invalid=N */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include "sq_oracle.h"

static uint64_t st = 88172645463325252ull;
static uint64_t nxt(void) { st ^= st << 13; st ^= st >> 7; st ^= st << 17; return st; }

static uint16_t rand_f16(int emin, int emax) { /* normal fp16 with exponent in [emin, emax] */
  int e = emin + (int)(nxt() % (uint64_t)(emax - emin + 1));
  return (uint16_t)(((e + 15) << 10) | (nxt() & 0x3ff));
}

int main(int argc, char** argv) {
  int trials = argc > 1 ? atoi(argv[1]) : 1;
  orc_layout L = {1, 4, 4, ORC_UNIT_HEAD, ORC_GATE_SCALAR, 2, 1, 0};
  uint8_t bits[1] = {2};
  size_t hb = orc_head_bytes(&L, bits, 0);
  long valid = 0, mismatch = 0, unstable = 0, checked_invalid = 0;
  uint8_t blk[64], blk2[64], blk3[64];
  float S[16];
  for (int t = 0; t < trials; ++t) {
    uint16_t r16[4], c16[4];
    int one_col = (int)(nxt() % 4);
    for (int i = 0; i < 4; ++i) r16[i] = rand_f16(-10, 2);
    for (int j = 0; j < 4; ++j) c16[j] = j == one_col ? 0x3c00 : rand_f16(-14, -1);
    for (long p = 0; p < 43046721L; ++p) {
      int code[16];
      long x = p;
      for (int e = 0; e < 16; ++e) { code[e] = (int)(x % 3) - 1; x /= 3; }
      int ok = 1;
      for (int i = 0; i < 4 && ok; ++i) {
        int row_ok = 0;
        for (int j = 0; j < 4; ++j) row_ok |= (code[i * 4 + j] != 0) && c16[j] == 0x3c00;
        ok = row_ok;
      }
      for (int j = 0; j < 4 && ok; ++j) {
        int col_ok = 0;
        for (int i = 0; i < 4; ++i) col_ok |= code[i * 4 + j] != 0;
        ok = col_ok;
      }
      if (!ok && (nxt() & 255)) continue; /* sample 1/256 of the invalid patterns */
      memset(blk, 0, sizeof blk);
      for (int i = 0; i < 4; ++i) { blk[2 * i] = r16[i] & 0xff; blk[2 * i + 1] = r16[i] >> 8; }
      for (int j = 0; j < 4; ++j) { blk[8 + 2 * j] = c16[j] & 0xff; blk[9 + 2 * j] = c16[j] >> 8; }
      for (int i = 0; i < 4; ++i) {
        int32_t u[4];
        for (int j = 0; j < 4; ++j) u[j] = code[i * 4 + j] + 2;
        orc_pack_row(2, 4, u, blk + 16 + i);
      }
      if (orc_dequantize_head(&L, bits, 0, blk, S)) { ++mismatch; continue; }
      if (orc_quantize_head(&L, bits, 0, S, blk2)) { ++mismatch; continue; }
      if (ok) {
        ++valid;
        if (memcmp(blk, blk2, hb)) ++mismatch;
      } else {
        ++checked_invalid;
        if (orc_dequantize_head(&L, bits, 0, blk2, S) || orc_quantize_head(&L, bits, 0, S, blk3) ||
            memcmp(blk2, blk3, hb))
          ++unstable;
      }
    }
  }
  printf("valid=%ld mismatch=%ld unstable=%ld checked_invalid=%ld\n", valid, mismatch, unstable,
         checked_invalid);
  return 0;
}
