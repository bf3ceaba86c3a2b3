// Packed-weight files: the offline packer's output stored once and loaded at
// serving time. Only the ternary weights are exported once training ends
// ("BitNet b1.58 2B4T Guide: Scaling Native 1-Bit LLMs", section
// "High-Precision Master Weights"), and the model ships pre-packed
// (winbuzzer.com release article, "Availability and Context"); this is the
// library's own container for its packed layout.
//
// File = 64-byte header + payload, all little-endian:
//   0  char[8]  magic "BITLIN58"
//   8  u32      format version (1)
//   12 u32      layout id (1: the 16-row-block, 128-k-group 2-bit layout of
//               include/bitlinear.h)
//   16 i64      N
//   24 i64      K
//   32 f32      gamma
//   36 u32      reserved, 0
//   40 u64      payload bytes (= bitlinear_packed_bytes(N, K))
//   48 u64      FNV-1a 64-bit hash of the payload
//   56 u64      reserved, 0
//   64 ...      payload
// Writes go to "<path>.tmp" and are renamed into place, so a reader never sees
// a half-written file under the final name.

#include <cstdint>
#include <cstdio>
#include <cstring>
#include <string>

#include "../../include/bitlinear.h"

namespace {

constexpr char kMagic[8] = {'B', 'I', 'T', 'L', 'I', 'N', '5', '8'};
constexpr uint32_t kVersion = 1;
constexpr uint32_t kLayout = 1;
constexpr size_t kHeaderBytes = 64;

// FNV-1a, 64-bit: offset basis 14695981039346656037, prime 1099511628211.
uint64_t fnv1a64(const uint8_t *p, size_t n, uint64_t h = 14695981039346656037ull)
{
    for (size_t i = 0; i < n; ++i) {
        h ^= p[i];
        h *= 1099511628211ull;
    }
    return h;
}

void put_u32(uint8_t *d, uint32_t v)
{
    for (int i = 0; i < 4; ++i)
        d[i] = static_cast<uint8_t>(v >> (8 * i));
}

void put_u64(uint8_t *d, uint64_t v)
{
    for (int i = 0; i < 8; ++i)
        d[i] = static_cast<uint8_t>(v >> (8 * i));
}

uint32_t get_u32(const uint8_t *s)
{
    uint32_t v = 0;
    for (int i = 0; i < 4; ++i)
        v |= static_cast<uint32_t>(s[i]) << (8 * i);
    return v;
}

uint64_t get_u64(const uint8_t *s)
{
    uint64_t v = 0;
    for (int i = 0; i < 8; ++i)
        v |= static_cast<uint64_t>(s[i]) << (8 * i);
    return v;
}

struct Header {
    int64_t N = 0, K = 0;
    float gamma = 0.0f;
    uint64_t payload = 0;
    uint64_t hash = 0;
};

// Reads and checks the header of an open file.
int read_header(FILE *f, Header *h)
{
    uint8_t b[kHeaderBytes];
    if (std::fread(b, 1, kHeaderBytes, f) != kHeaderBytes)
        return BITLINEAR_ERR_FORMAT;
    if (std::memcmp(b, kMagic, 8) != 0 || get_u32(b + 8) != kVersion ||
        get_u32(b + 12) != kLayout)
        return BITLINEAR_ERR_FORMAT;
    h->N = static_cast<int64_t>(get_u64(b + 16));
    h->K = static_cast<int64_t>(get_u64(b + 24));
    const uint32_t gbits = get_u32(b + 32);
    std::memcpy(&h->gamma, &gbits, 4);
    h->payload = get_u64(b + 40);
    h->hash = get_u64(b + 48);
    if (bitlinear_packed_bytes(h->N, h->K) == 0 || h->payload != bitlinear_packed_bytes(h->N, h->K))
        return BITLINEAR_ERR_FORMAT;
    if (!(h->gamma > 0.0f) || !(h->gamma <= 3.4e38f))
        return BITLINEAR_ERR_FORMAT;
    return BITLINEAR_OK;
}

}  // namespace

extern "C" int bitlinear_save_packed(const char *path, const void *packed_host, int64_t N,
                                     int64_t K, float gamma)
{
    if (path == nullptr || packed_host == nullptr)
        return BITLINEAR_ERR_ARG;
    const size_t bytes = bitlinear_packed_bytes(N, K);
    if (bytes == 0)
        return BITLINEAR_ERR_SHAPE;
    if (!(gamma > 0.0f) || !(gamma <= 3.4e38f))
        return BITLINEAR_ERR_ARG;
    const uint8_t *payload = static_cast<const uint8_t *>(packed_host);
    uint8_t b[kHeaderBytes] = {};
    std::memcpy(b, kMagic, 8);
    put_u32(b + 8, kVersion);
    put_u32(b + 12, kLayout);
    put_u64(b + 16, static_cast<uint64_t>(N));
    put_u64(b + 24, static_cast<uint64_t>(K));
    uint32_t gbits;
    std::memcpy(&gbits, &gamma, 4);
    put_u32(b + 32, gbits);
    put_u64(b + 40, bytes);
    put_u64(b + 48, fnv1a64(payload, bytes));

    std::string tmp;
    try {
        tmp = std::string(path) + ".tmp";
    } catch (...) {
        return BITLINEAR_ERR_HOST;
    }
    FILE *f = std::fopen(tmp.c_str(), "wb");
    if (f == nullptr)
        return BITLINEAR_ERR_IO;
    bool ok = std::fwrite(b, 1, kHeaderBytes, f) == kHeaderBytes &&
              std::fwrite(payload, 1, bytes, f) == bytes;
    ok = (std::fclose(f) == 0) && ok;
    if (!ok || std::rename(tmp.c_str(), path) != 0) {
        std::remove(tmp.c_str());
        return BITLINEAR_ERR_IO;
    }
    return BITLINEAR_OK;
}

extern "C" int bitlinear_read_packed_header(const char *path, int64_t *N_out, int64_t *K_out,
                                            float *gamma_out)
{
    if (path == nullptr || N_out == nullptr || K_out == nullptr || gamma_out == nullptr)
        return BITLINEAR_ERR_ARG;
    FILE *f = std::fopen(path, "rb");
    if (f == nullptr)
        return BITLINEAR_ERR_IO;
    Header h;
    const int rc = read_header(f, &h);
    std::fclose(f);
    if (rc != BITLINEAR_OK)
        return rc;
    *N_out = h.N;
    *K_out = h.K;
    *gamma_out = h.gamma;
    return BITLINEAR_OK;
}

extern "C" int bitlinear_load_packed(const char *path, void *packed_host, size_t packed_bytes,
                                     int64_t *N_out, int64_t *K_out, float *gamma_out)
{
    if (path == nullptr || packed_host == nullptr || N_out == nullptr || K_out == nullptr ||
        gamma_out == nullptr)
        return BITLINEAR_ERR_ARG;
    FILE *f = std::fopen(path, "rb");
    if (f == nullptr)
        return BITLINEAR_ERR_IO;
    Header h;
    int rc = read_header(f, &h);
    if (rc == BITLINEAR_OK && packed_bytes < h.payload)
        rc = BITLINEAR_ERR_ARG;
    uint8_t *dst = static_cast<uint8_t *>(packed_host);
    if (rc == BITLINEAR_OK && std::fread(dst, 1, h.payload, f) != h.payload)
        rc = BITLINEAR_ERR_FORMAT;                      // truncated payload
    if (rc == BITLINEAR_OK && std::fgetc(f) != EOF)
        rc = BITLINEAR_ERR_FORMAT;                      // trailing bytes
    std::fclose(f);
    if (rc == BITLINEAR_OK && fnv1a64(dst, h.payload) != h.hash)
        rc = BITLINEAR_ERR_FORMAT;                      // corrupted payload
    if (rc != BITLINEAR_OK)
        return rc;
    *N_out = h.N;
    *K_out = h.K;
    *gamma_out = h.gamma;
    return BITLINEAR_OK;
}
