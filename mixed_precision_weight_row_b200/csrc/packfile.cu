// On-disk container for packed matrices (host code, no device work).
//
// DynaQuant, "Status": bit pack / unpack tools are done, a packed weight
// format for disk storage is in progress.  This is that format for the rows
// this library packs:
//
//   header (32 bytes)   magic "MPWPACK\0", u32 version (1), u32 count,
//                       u64 index offset (32), u64 data offset
//   index (64 bytes per matrix)
//                       u64 N, u64 K, u32 bits, u32 layout,
//                       u64 packed offset, u64 packed bytes (N * row bytes),
//                       u64 scales offset, u32 CRC-32 of the packed bytes,
//                       u32 CRC-32 of the scales, u64 reserved (0)
//   data                per matrix the packed rows, then the fp32 scales,
//                       each starting at a multiple of 64 bytes (zero fill)
//
// All integers and the scales little-endian (the host's order).  CRC-32 is
// the IEEE 802.3 checksum (reflected polynomial 0xEDB88320, initial value and
// final XOR 0xFFFFFFFF).
#include <stdint.h>

#include <cstdio>
#include <cstring>
#include <vector>

#include "mpw.h"

namespace {

constexpr char kMagic[8] = {'M', 'P', 'W', 'P', 'A', 'C', 'K', '\0'};
constexpr uint32_t kVersion = 1;
constexpr uint64_t kHeaderBytes = 32;
constexpr uint64_t kEntryBytes = 64;
constexpr uint64_t kAlign = 64;

struct CrcTable {
  uint32_t t[256];
  CrcTable() {
    for (uint32_t i = 0; i < 256; ++i) {
      uint32_t c = i;
      for (int k = 0; k < 8; ++k) c = (c & 1u) ? (0xEDB88320u ^ (c >> 1)) : (c >> 1);
      t[i] = c;
    }
  }
};

uint32_t crc32_update(uint32_t crc, const uint8_t* p, size_t n) {
  static const CrcTable tab;  // initialised once, thread-safe
  const uint32_t* table = tab.t;
  crc = ~crc;
  for (size_t i = 0; i < n; ++i) crc = table[(crc ^ p[i]) & 0xFFu] ^ (crc >> 8);
  return ~crc;
}

uint64_t align_up(uint64_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

uint64_t row_bytes(int64_t K, int bits) {
  return 16u * ((static_cast<uint64_t>(K) * static_cast<uint64_t>(bits) + 127u) / 128u);
}

void put_u32(uint8_t* p, uint32_t v) {
  for (int i = 0; i < 4; ++i) p[i] = static_cast<uint8_t>(v >> (8 * i));
}
void put_u64(uint8_t* p, uint64_t v) {
  for (int i = 0; i < 8; ++i) p[i] = static_cast<uint8_t>(v >> (8 * i));
}
uint32_t get_u32(const uint8_t* p) {
  uint32_t v = 0;
  for (int i = 3; i >= 0; --i) v = (v << 8) | p[i];
  return v;
}
uint64_t get_u64(const uint8_t* p) {
  uint64_t v = 0;
  for (int i = 7; i >= 0; --i) v = (v << 8) | p[i];
  return v;
}

struct Entry {
  uint64_t N, K;
  uint32_t bits, layout;
  uint64_t packed_off, packed_bytes, scales_off;
  uint32_t crc_packed, crc_scales;
};

bool valid_shape(int64_t N, int64_t K, int bits, int layout) {
  if (N < 1 || K < 1 || N >= (int64_t{1} << 31) || K >= (int64_t{1} << 31)) return false;
  if (bits < 4 || bits > 15) return false;
  if (layout != MPW_LAYOUT_CANONICAL && layout != MPW_LAYOUT_PAIRED) return false;
  return layout != MPW_LAYOUT_PAIRED || K % 32 == 0;
}

struct File {
  FILE* f = nullptr;
  ~File() {
    if (f != nullptr) fclose(f);
  }
};

uint64_t file_size(FILE* f) {
  if (fseek(f, 0, SEEK_END) != 0) return 0;
  const long n = ftell(f);
  return n < 0 ? 0 : static_cast<uint64_t>(n);
}

bool read_at(FILE* f, uint64_t off, void* dst, size_t n) {
  return fseek(f, static_cast<long>(off), SEEK_SET) == 0 && fread(dst, 1, n, f) == n;
}

// Reads and checks the header and the index; MPW_E_IO if the file cannot be
// read, MPW_E_FORMAT if it is not a valid container.
mpw_status load_index(const char* path, File& file, std::vector<Entry>& out) {
  file.f = fopen(path, "rb");
  if (file.f == nullptr) return MPW_E_IO;
  const uint64_t size = file_size(file.f);
  uint8_t h[kHeaderBytes];
  if (size < kHeaderBytes || !read_at(file.f, 0, h, sizeof(h))) return MPW_E_FORMAT;
  if (std::memcmp(h, kMagic, 8) != 0 || get_u32(h + 8) != kVersion) return MPW_E_FORMAT;
  const uint32_t count = get_u32(h + 12);
  const uint64_t index_off = get_u64(h + 16), data_off = get_u64(h + 24);
  if (index_off != kHeaderBytes || count > (1u << 24)) return MPW_E_FORMAT;
  if (index_off + static_cast<uint64_t>(count) * kEntryBytes > data_off || data_off > size) return MPW_E_FORMAT;
  std::vector<uint8_t> idx(static_cast<size_t>(count) * kEntryBytes);
  if (count > 0 && !read_at(file.f, index_off, idx.data(), idx.size())) return MPW_E_FORMAT;
  out.resize(count);
  for (uint32_t i = 0; i < count; ++i) {
    const uint8_t* p = idx.data() + static_cast<size_t>(i) * kEntryBytes;
    Entry& e = out[i];
    e.N = get_u64(p);
    e.K = get_u64(p + 8);
    e.bits = get_u32(p + 16);
    e.layout = get_u32(p + 20);
    e.packed_off = get_u64(p + 24);
    e.packed_bytes = get_u64(p + 32);
    e.scales_off = get_u64(p + 40);
    e.crc_packed = get_u32(p + 48);
    e.crc_scales = get_u32(p + 52);
    if (!valid_shape(static_cast<int64_t>(e.N), static_cast<int64_t>(e.K), static_cast<int>(e.bits),
                     static_cast<int>(e.layout)))
      return MPW_E_FORMAT;
    if (e.packed_bytes != e.N * row_bytes(static_cast<int64_t>(e.K), static_cast<int>(e.bits))) return MPW_E_FORMAT;
    if (e.packed_off < data_off || e.packed_off + e.packed_bytes > size) return MPW_E_FORMAT;
    if (e.scales_off < data_off || e.scales_off + 4u * e.N > size) return MPW_E_FORMAT;
  }
  return MPW_OK;
}

}  // namespace

extern "C" {

mpw_status mpw_file_write(const char* path, const mpw_file_matrix* m, int64_t count) {
  if (path == nullptr || m == nullptr || count < 1 || count > (1 << 24)) return MPW_E_INVALID_ARG;
  for (int64_t i = 0; i < count; ++i) {
    if (m[i].bits < 4 || m[i].bits > 15) return MPW_E_UNSUPPORTED_BITS;
    if (m[i].packed == nullptr || m[i].scales == nullptr || !valid_shape(m[i].N, m[i].K, m[i].bits, m[i].layout))
      return MPW_E_INVALID_ARG;
  }
  // lay out the data
  std::vector<Entry> es(static_cast<size_t>(count));
  uint64_t off = align_up(kHeaderBytes + static_cast<uint64_t>(count) * kEntryBytes);
  const uint64_t data_off = off;
  for (int64_t i = 0; i < count; ++i) {
    Entry& e = es[static_cast<size_t>(i)];
    e.N = static_cast<uint64_t>(m[i].N);
    e.K = static_cast<uint64_t>(m[i].K);
    e.bits = static_cast<uint32_t>(m[i].bits);
    e.layout = static_cast<uint32_t>(m[i].layout);
    e.packed_bytes = e.N * row_bytes(m[i].K, m[i].bits);
    e.packed_off = off;
    off = align_up(off + e.packed_bytes);
    e.scales_off = off;
    off = align_up(off + 4u * e.N);
    e.crc_packed = crc32_update(0u, m[i].packed, static_cast<size_t>(e.packed_bytes));
    e.crc_scales = crc32_update(0u, reinterpret_cast<const uint8_t*>(m[i].scales), static_cast<size_t>(4u * e.N));
  }
  std::vector<uint8_t> head(static_cast<size_t>(data_off), 0);
  std::memcpy(head.data(), kMagic, 8);
  put_u32(head.data() + 8, kVersion);
  put_u32(head.data() + 12, static_cast<uint32_t>(count));
  put_u64(head.data() + 16, kHeaderBytes);
  put_u64(head.data() + 24, data_off);
  for (int64_t i = 0; i < count; ++i) {
    uint8_t* p = head.data() + kHeaderBytes + static_cast<size_t>(i) * kEntryBytes;
    const Entry& e = es[static_cast<size_t>(i)];
    put_u64(p, e.N);
    put_u64(p + 8, e.K);
    put_u32(p + 16, e.bits);
    put_u32(p + 20, e.layout);
    put_u64(p + 24, e.packed_off);
    put_u64(p + 32, e.packed_bytes);
    put_u64(p + 40, e.scales_off);
    put_u32(p + 48, e.crc_packed);
    put_u32(p + 52, e.crc_scales);
  }
  File file;
  file.f = fopen(path, "wb");
  if (file.f == nullptr) return MPW_E_IO;
  if (fwrite(head.data(), 1, head.size(), file.f) != head.size()) return MPW_E_IO;
  static const uint8_t zeros[kAlign] = {};
  uint64_t at = data_off;
  auto write_blob = [&](uint64_t where, const void* p, uint64_t n) {
    if (where > at && fwrite(zeros, 1, static_cast<size_t>(where - at), file.f) != where - at) return false;
    if (fwrite(p, 1, static_cast<size_t>(n), file.f) != n) return false;
    at = where + n;
    return true;
  };
  for (int64_t i = 0; i < count; ++i) {
    const Entry& e = es[static_cast<size_t>(i)];
    if (!write_blob(e.packed_off, m[i].packed, e.packed_bytes)) return MPW_E_IO;
    if (!write_blob(e.scales_off, m[i].scales, 4u * e.N)) return MPW_E_IO;
  }
  if (off > at && fwrite(zeros, 1, static_cast<size_t>(off - at), file.f) != off - at) return MPW_E_IO;
  if (fflush(file.f) != 0) return MPW_E_IO;
  return MPW_OK;
}

mpw_status mpw_file_count(const char* path, int64_t* count) {
  if (path == nullptr || count == nullptr) return MPW_E_INVALID_ARG;
  File file;
  std::vector<Entry> es;
  const mpw_status st = load_index(path, file, es);
  if (st != MPW_OK) return st;
  *count = static_cast<int64_t>(es.size());
  return MPW_OK;
}

mpw_status mpw_file_info(const char* path, int64_t index, int64_t* N, int64_t* K, int32_t* bits, int32_t* layout) {
  if (path == nullptr || N == nullptr || K == nullptr || bits == nullptr || layout == nullptr || index < 0)
    return MPW_E_INVALID_ARG;
  File file;
  std::vector<Entry> es;
  const mpw_status st = load_index(path, file, es);
  if (st != MPW_OK) return st;
  if (index >= static_cast<int64_t>(es.size())) return MPW_E_INVALID_ARG;
  const Entry& e = es[static_cast<size_t>(index)];
  *N = static_cast<int64_t>(e.N);
  *K = static_cast<int64_t>(e.K);
  *bits = static_cast<int32_t>(e.bits);
  *layout = static_cast<int32_t>(e.layout);
  return MPW_OK;
}

mpw_status mpw_file_read(const char* path, int64_t index, uint8_t* packed, float* scales) {
  if (path == nullptr || packed == nullptr || scales == nullptr || index < 0) return MPW_E_INVALID_ARG;
  File file;
  std::vector<Entry> es;
  const mpw_status st = load_index(path, file, es);
  if (st != MPW_OK) return st;
  if (index >= static_cast<int64_t>(es.size())) return MPW_E_INVALID_ARG;
  const Entry& e = es[static_cast<size_t>(index)];
  if (!read_at(file.f, e.packed_off, packed, static_cast<size_t>(e.packed_bytes))) return MPW_E_FORMAT;
  if (!read_at(file.f, e.scales_off, scales, static_cast<size_t>(4u * e.N))) return MPW_E_FORMAT;
  if (crc32_update(0u, packed, static_cast<size_t>(e.packed_bytes)) != e.crc_packed ||
      crc32_update(0u, reinterpret_cast<const uint8_t*>(scales), static_cast<size_t>(4u * e.N)) != e.crc_scales)
    return MPW_E_FORMAT;
  return MPW_OK;
}

}  // extern "C"
