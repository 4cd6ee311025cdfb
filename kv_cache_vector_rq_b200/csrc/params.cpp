// Parameter files (host): the seed-derived parameters of one configuration written to a
// file and read back with a checksum.
//
// The parameters are a pure function of (d, bits, m, seed) -- "TurboQuant 论文解读",
// "简单复现 demo" (a fixed random rotation and Gaussian projection), "TurboQuant +
// RotorQuant", "How RotorQuant Works" (random unit rotors), "Codebook Calibration Fix"
// (the Lloyd-Max codebook of the rotated-coordinate density) -- so a file is a record of
// them, for reproducibility or for a process without the setup code. Layout:
//   line 1  "KVRQ-PARAMS 1"
//   line 2  a JSON object: {"d": .., "bits": .., "m": .., "seed": .., "rotors": n, "pi": n,
//           "T": n, "centroids": n, "fnv1a64": "<16 hex digits>"}
//   then    the float64 arrays, little-endian, in that order: rotors [G][4] (stream seed + 1),
//           pi [d][d] (seed + 2), T [m][d] (seed + 3), centroids [2^bits].
// The checksum is FNV-1a (64-bit) over the payload bytes.

#include <cinttypes>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "kvrq.h"
#include "kvrq_internal.h"

using namespace kvrq;

namespace {

constexpr const char* kMagic = "KVRQ-PARAMS 1";

uint64_t fnv1a64(const void* data, size_t bytes, uint64_t h = 1469598103934665603ull) {
  const uint8_t* p = static_cast<const uint8_t*>(data);
  for (size_t i = 0; i < bytes; ++i) {
    h ^= p[i];
    h *= 1099511628211ull;
  }
  return h;
}

// Value of the integer field "key" in a one-line JSON object; false if absent.
bool json_int(const std::string& line, const char* key, long long* out) {
  const std::string k = std::string("\"") + key + "\":";
  const size_t at = line.find(k);
  if (at == std::string::npos) return false;
  return std::sscanf(line.c_str() + at + k.size(), " %lld", out) == 1;
}

bool json_u64(const std::string& line, const char* key, uint64_t* out) {
  const std::string k = std::string("\"") + key + "\":";
  const size_t at = line.find(k);
  if (at == std::string::npos) return false;
  unsigned long long v = 0;
  if (std::sscanf(line.c_str() + at + k.size(), " %llu", &v) != 1) return false;
  *out = (uint64_t)v;
  return true;
}

bool json_hex(const std::string& line, const char* key, uint64_t* out) {
  const std::string k = std::string("\"") + key + "\":";
  const size_t at = line.find(k);
  if (at == std::string::npos) return false;
  unsigned long long v = 0;
  if (std::sscanf(line.c_str() + at + k.size(), " \"%16llx\"", &v) != 1) return false;
  *out = (uint64_t)v;
  return true;
}

struct Sizes {
  int64_t rotors, pi, T, centroids;
  int64_t total() const { return rotors + pi + T + centroids; }
};

Sizes sizes_of(int d, int bits, int m) { return {4 * (int64_t)((d + 2) / 3), (int64_t)d * d, (int64_t)m * d, (int64_t)1 << bits}; }

kvrq_status check_config(const char* name, int d, int bits, int m) {
  if (d < 2 || d > 16384 || bits < 1 || bits > 8 || m < 1 || m > 16384)
    return set_errorf(KVRQ_EINVAL, "%s: 2 <= d <= 16384, 1 <= bits <= 8, 1 <= m <= 16384", name);
  return KVRQ_OK;
}

}  // namespace

extern "C" {

kvrq_status kvrq_params_export(const char* path, int d, int bits, int m, uint64_t seed) {
  const char* name = "kvrq_params_export";
  if (!path) return set_error(KVRQ_EINVAL, "kvrq_params_export: path is NULL");
  kvrq_status st = check_config(name, d, bits, m);
  if (st != KVRQ_OK) return st;
  return guarded(name, [&]() -> kvrq_status {
    alloc_check();
    const Sizes sz = sizes_of(d, bits, m);
    std::vector<double> payload((size_t)sz.total());
    double* rot = payload.data();
    double* pi = rot + sz.rotors;
    double* T = pi + sz.pi;
    double* c = T + sz.T;
    kvrq_status s2;
    if ((s2 = rq_rotors_init(d, seed + 1, rot)) != KVRQ_OK) return s2;
    if ((s2 = tq_rotation_init(d, seed + 2, pi)) != KVRQ_OK) return s2;
    if ((s2 = qjl_matrix_init(m, d, seed + 3, T)) != KVRQ_OK) return s2;
    if ((s2 = tq_codebook_init(d, bits, 1e-13, 100000, c, nullptr, nullptr)) != KVRQ_OK) return s2;
    const uint64_t h = fnv1a64(payload.data(), payload.size() * sizeof(double));
    FILE* f = std::fopen(path, "wb");
    if (!f) return set_errorf(KVRQ_EINVAL, "%s: cannot open %s for writing", name, path);
    std::fprintf(f, "%s\n{\"d\": %d, \"bits\": %d, \"m\": %d, \"seed\": %" PRIu64 ", \"rotors\": %" PRId64
                 ", \"pi\": %" PRId64 ", \"T\": %" PRId64 ", \"centroids\": %" PRId64 ", \"fnv1a64\": \"%016" PRIx64
                 "\"}\n",
                 kMagic, d, bits, m, seed, sz.rotors, sz.pi, sz.T, sz.centroids, h);
    const size_t wrote = std::fwrite(payload.data(), sizeof(double), payload.size(), f);
    const bool ok = std::fclose(f) == 0 && wrote == payload.size();
    if (!ok) return set_errorf(KVRQ_EINVAL, "%s: writing %s failed", name, path);
    return KVRQ_OK;
  });
}

kvrq_status kvrq_params_import(const char* path, int d, int bits, int m, uint64_t* seed, double* rotors, double* pi,
                               double* T, double* centroids) {
  const char* name = "kvrq_params_import";
  if (!path) return set_error(KVRQ_EINVAL, "kvrq_params_import: path is NULL");
  kvrq_status st = check_config(name, d, bits, m);
  if (st != KVRQ_OK) return st;
  return guarded(name, [&]() -> kvrq_status {
    alloc_check();
    FILE* f = std::fopen(path, "rb");
    if (!f) return set_errorf(KVRQ_EINVAL, "%s: cannot open %s", name, path);
    std::vector<char> buf(4096);
    std::string magic, header;
    if (std::fgets(buf.data(), (int)buf.size(), f)) magic = buf.data();
    if (std::fgets(buf.data(), (int)buf.size(), f)) header = buf.data();
    if (magic != std::string(kMagic) + "\n") {
      std::fclose(f);
      return set_errorf(KVRQ_EINVAL, "%s: %s is not a parameter file", name, path);
    }
    long long fd = 0, fb = 0, fm = 0, nr = 0, np = 0, nt = 0, nc = 0;
    uint64_t h = 0, fs = 0;
    if (!json_int(header, "d", &fd) || !json_int(header, "bits", &fb) || !json_int(header, "m", &fm) ||
        !json_u64(header, "seed", &fs) || !json_int(header, "rotors", &nr) || !json_int(header, "pi", &np) ||
        !json_int(header, "T", &nt) || !json_int(header, "centroids", &nc) || !json_hex(header, "fnv1a64", &h)) {
      std::fclose(f);
      return set_errorf(KVRQ_EINVAL, "%s: malformed header in %s", name, path);
    }
    const Sizes sz = sizes_of(d, bits, m);
    if (fd != d || fb != bits || fm != m || nr != sz.rotors || np != sz.pi || nt != sz.T || nc != sz.centroids) {
      std::fclose(f);
      return set_errorf(KVRQ_EINVAL, "%s: %s holds d = %lld, bits = %lld, m = %lld, not the configuration asked for",
                        name, path, fd, fb, fm);
    }
    std::vector<double> payload((size_t)sz.total());
    const size_t got = std::fread(payload.data(), sizeof(double), payload.size(), f);
    const bool extra = std::fgetc(f) != EOF;
    std::fclose(f);
    if (got != payload.size() || extra) return set_errorf(KVRQ_EINVAL, "%s: %s has the wrong length", name, path);
    if (fnv1a64(payload.data(), payload.size() * sizeof(double)) != h)
      return set_errorf(KVRQ_ECHECKSUM, "%s: the contents of %s do not match its checksum", name, path);
    const double* p = payload.data();
    if (rotors) std::memcpy(rotors, p, (size_t)sz.rotors * sizeof(double));
    p += sz.rotors;
    if (pi) std::memcpy(pi, p, (size_t)sz.pi * sizeof(double));
    p += sz.pi;
    if (T) std::memcpy(T, p, (size_t)sz.T * sizeof(double));
    p += sz.T;
    if (centroids) std::memcpy(centroids, p, (size_t)sz.centroids * sizeof(double));
    if (seed) *seed = fs;
    return KVRQ_OK;
  });
}

}  // extern "C"
