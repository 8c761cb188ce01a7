// The one persistent artefact of the method: the Smooth-QK calibration.  The HiFA4
// abstract fixes the per-channel scales offline ("calibration-static"), so a deployment
// computes them once (hifa4_calibrate_smooth) and loads them with the model.  File
// layout, little-endian, no padding:
//   bytes  0..7   magic "HIFA4CAL"
//   bytes  8..11  version (uint32) = 1
//   bytes 12..15  Hkv (int32)     bytes 16..19  d (int32)
//   bytes 20..23  alpha (fp32)    bytes 24..27  CRC-32 (IEEE 802.3) of the two arrays
//   then s [Hkv * d] fp32, then s_inv [Hkv * d] fp32.
#include <cstdio>
#include <cstring>
#include <vector>

#include "../../include/hifa4.h"

namespace {

const char kMagic[8] = {'H', 'I', 'F', 'A', '4', 'C', 'A', 'L'};
constexpr uint32_t kVersion = 1;

uint32_t crc32_ieee(const unsigned char* p, size_t n, uint32_t crc = 0) {
  crc = ~crc;
  for (size_t i = 0; i < n; ++i) {
    crc ^= p[i];
    for (int k = 0; k < 8; ++k) crc = (crc >> 1) ^ (0xEDB88320u & (0u - (crc & 1u)));
  }
  return ~crc;
}

bool little_endian() {
  const uint32_t one = 1;
  unsigned char c;
  std::memcpy(&c, &one, 1);
  return c == 1;
}

void put_u32(unsigned char* p, uint32_t v) {
  for (int i = 0; i < 4; ++i) p[i] = (unsigned char)(v >> (8 * i));
}
uint32_t get_u32(const unsigned char* p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
uint32_t f32_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}
float bits_f32(uint32_t u) {
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

}  // namespace

extern "C" {

int hifa4_calibration_save(const char* path, int Hkv, int d, float alpha, const float* s, const float* sinv) {
  if (!path || !s || !sinv || Hkv <= 0 || d <= 0 || Hkv > (1 << 20) || d > 4096 || !(alpha >= 0.0f))
    return HIFA4_ERR_INVALID_ARG;
  if (!little_endian()) return HIFA4_ERR_IO;
  const size_t n = (size_t)Hkv * d;
  std::vector<unsigned char> body(8 * n);
  for (size_t i = 0; i < n; ++i) put_u32(&body[4 * i], f32_bits(s[i]));
  for (size_t i = 0; i < n; ++i) put_u32(&body[4 * (n + i)], f32_bits(sinv[i]));
  unsigned char head[28];
  std::memcpy(head, kMagic, 8);
  put_u32(head + 8, kVersion);
  put_u32(head + 12, (uint32_t)Hkv);
  put_u32(head + 16, (uint32_t)d);
  put_u32(head + 20, f32_bits(alpha));
  put_u32(head + 24, crc32_ieee(body.data(), body.size()));
  FILE* f = std::fopen(path, "wb");
  if (!f) return HIFA4_ERR_IO;
  const bool ok = std::fwrite(head, 1, 28, f) == 28 && std::fwrite(body.data(), 1, body.size(), f) == body.size();
  return (std::fclose(f) == 0 && ok) ? HIFA4_OK : HIFA4_ERR_IO;
}

int hifa4_calibration_load(const char* path, int* Hkv, int* d, float* alpha, float* s, float* sinv,
                           size_t capacity) {
  if (!path || !Hkv || !d || !alpha) return HIFA4_ERR_INVALID_ARG;
  FILE* f = std::fopen(path, "rb");
  if (!f) return HIFA4_ERR_IO;
  unsigned char head[28];
  if (std::fread(head, 1, 28, f) != 28 || std::memcmp(head, kMagic, 8) != 0 || get_u32(head + 8) != kVersion) {
    std::fclose(f);
    return HIFA4_ERR_IO;
  }
  const int hk = (int)get_u32(head + 12), dd = (int)get_u32(head + 16);
  if (hk <= 0 || dd <= 0 || hk > (1 << 20) || dd > 4096) {
    std::fclose(f);
    return HIFA4_ERR_IO;
  }
  *Hkv = hk;
  *d = dd;
  *alpha = bits_f32(get_u32(head + 20));
  const size_t n = (size_t)hk * dd;
  if (!s || !sinv || capacity < n) {   // header only: the caller sizes its arrays and calls again
    std::fclose(f);
    return (s || sinv) ? HIFA4_ERR_INVALID_ARG : HIFA4_OK;
  }
  std::vector<unsigned char> body(8 * n);
  const bool got = std::fread(body.data(), 1, body.size(), f) == body.size();
  unsigned char extra;
  const bool at_end = got && std::fread(&extra, 1, 1, f) == 0;
  std::fclose(f);
  if (!got || !at_end || crc32_ieee(body.data(), body.size()) != get_u32(head + 24)) return HIFA4_ERR_IO;
  for (size_t i = 0; i < n; ++i) s[i] = bits_f32(get_u32(&body[4 * i]));
  for (size_t i = 0; i < n; ++i) sinv[i] = bits_f32(get_u32(&body[4 * (n + i)]));
  return HIFA4_OK;
}

}  // extern "C"
