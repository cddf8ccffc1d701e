// Device table block of the hx library (private to the library; HX_TABLES_BYTES bytes).
// Written on the host by hx_codebook_tables / hx_codebook_upload, read by the kernels.
#pragma once
#include <stdint.h>

#include "hx.h"

namespace hx {

constexpr uint32_t kTablesMagic = 0x42545848u;  // "HXTB"
// Set in every decode table entry that holds a code word: a decoder ANDs the entries it uses and
// finds an unused window (entry 0) from one bit at the end.
constexpr uint32_t kDecValid = 0x10u;

struct Tables {
  // Encoder: per byte value (code << 4) | len; len 0 = no code word.
  uint32_t enc[256];
  union {
    // Decoder: for every 12-bit window w, (sym << 8) | kDecValid | len of the code word that w
    // starts with; 0 when no code word is a prefix of w. (Filled for QLC codebooks as well.)
    uint16_t dec[4096];
    // Shannonic (kind 2) instead:
    struct {
      // per decoding state 128 + u, four words: the mask of the bits its symbol took (the
      // offset and the state bits, 2^(nb + ob) - 1); their count nb + ob; nb (bits 0-4) | the
      // base of the next state (xs << nb, bits 16-23: the next state is base + the nb state
      // bits); first byte value of the range (bits 0-15) | 0x8000 - range size (16-31), so that
      // offset * 0x10001 + this word holds the byte in bits 0-7 and sets bit 31 exactly when the
      // offset is not inside the range
      uint32_t sh_dec[128][4];
      // per byte value: offset bits ob (bits 0-3) | cum_r - f_r + 128 (8-15) | the 12-bit key
      // 256 * ob + (k << 8) - (f_r << k), k = 7 - floor(log2 f_r) (20-31): for a state x in
      // [128, 256), (x + key) >> 8 = nb + ob, nb the state bits the step writes (x >> nb in
      // [f_r, 2 f_r))
      uint32_t sh_sym[256];
      // per byte value: its offset in its range
      uint8_t sh_off[256];
      // the ranges' decoding states in increasing order (128 + u), ranges one after another
      uint8_t sh_enc[128];
    };
  };
  // QLC: byte value of each rank.
  uint8_t rank2sym[256];
  // QLC area a: first rank (bits 0-8) | number of ranks it holds (bits 9-17) | index bits (18-21).
  uint32_t qlc_area[8];
  // QLC: index bits of area a in nibble a.
  uint32_t qlc_bits_packed;
  uint32_t kind;
  uint32_t lmax;
  uint32_t magic;
  // 1 when every 12-bit window starts with a code word (Kraft sum 1): decode needs no check
  // for unused code words.
  uint32_t complete;
  uint64_t hash;
};

static_assert(sizeof(Tables) <= HX_TABLES_BYTES, "table block too large");
static_assert(offsetof(Tables, dec) % 16 == 0, "decode table must be 16-byte aligned");

}  // namespace hx
