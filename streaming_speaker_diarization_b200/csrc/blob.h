// Host-side helpers shared by the engines: the SFW1 weight container
// (parsed in place: tensor names, shapes and float32 payloads) and bf16
// rounding of weights at load time.
#pragma once
#include <stdint.h>
#include <string.h>

#include <string>
#include <unordered_map>
#include <vector>

namespace sf {

// ------------------------------------------------------------------ utils
inline uint16_t f2bf_bits(float f) {   // round to nearest even
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)((u >> 16) | ((u & 0xffff) ? 0x40 : 0));
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

struct TensorRef {
  const float* data = nullptr;
  std::vector<uint32_t> shape;
  size_t numel() const {
    size_t n = 1;
    for (auto d : shape) n *= d;
    return n;
  }
};


// ------------------------------------------------------------ blob parsing
inline bool parse_blob(const void* blob, uint64_t n, std::unordered_map<std::string, TensorRef>& out, std::string& err) {
  const uint8_t* b = static_cast<const uint8_t*>(blob);
  if (n < 16 || memcmp(b, "SFW1", 4) != 0) { err = "weight blob: bad magic"; return false; }
  uint32_t cnt;
  uint64_t data_off;
  memcpy(&cnt, b + 4, 4);
  memcpy(&data_off, b + 8, 8);
  size_t pos = 16;
  for (uint32_t i = 0; i < cnt; ++i) {
    if (pos + 2 > n) { err = "weight blob: truncated header"; return false; }
    uint16_t nl;
    memcpy(&nl, b + pos, 2);
    pos += 2;
    if (pos + nl + 1 > n) { err = "weight blob: truncated name"; return false; }
    std::string name(reinterpret_cast<const char*>(b + pos), nl);
    pos += nl;
    uint8_t nd = b[pos++];
    TensorRef t;
    for (int d = 0; d < nd; ++d) {
      uint32_t v;
      if (pos + 4 > n) { err = "weight blob: truncated dims"; return false; }
      memcpy(&v, b + pos, 4);
      pos += 4;
      t.shape.push_back(v);
    }
    uint64_t off;
    if (pos + 8 > n) { err = "weight blob: truncated offset"; return false; }
    memcpy(&off, b + pos, 8);
    pos += 8;
    if (data_off + off + t.numel() * 4 > n) { err = "weight blob: payload of " + name + " out of range"; return false; }
    t.data = reinterpret_cast<const float*>(b + data_off + off);
    out[name] = t;
  }
  return true;
}

struct Loader {
  std::unordered_map<std::string, TensorRef>& m;
  std::string err;
  const float* get(const std::string& name, std::vector<uint32_t> shape) {
    auto it = m.find(name);
    if (it == m.end()) {
      if (err.empty()) err = "weight blob: missing tensor " + name;
      return nullptr;
    }
    if (it->second.shape != shape) {
      if (err.empty()) err = "weight blob: tensor " + name + " has an unexpected shape";
      return nullptr;
    }
    return it->second.data;
  }
};

}  // namespace sf
