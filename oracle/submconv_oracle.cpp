// C++ CPU oracle for SubMConv3d.  TEST INFRASTRUCTURE ONLY: it is built and
// loaded by the tests and by the CPU baseline of the benchmark, never by the
// product library, and it shares no code with it.
//
// Definition followed (trellis_sparse_mlx README, "What's in it" and
// "Correctness"): for every active voxel c, out[c] = sum over kernel offsets d
// of feats[c + stride*d] @ W[d], taken over active neighbours only, with the
// output sites equal to the input sites.  Offsets are enumerated with x
// slowest: k = ((dx + r) * K + (dy + r)) * K + (dz + r), r = K / 2.
// Voxels of different batch index are never neighbours; a missing neighbour
// is -1 in the neighbour map; duplicate coordinates are an error.
//
// The coordinate dictionary is a std::unordered_map keyed by the four int32
// fields themselves; accumulation is in double over inputs already rounded to
// the workload dtype.  OpenMP parallelises over voxels only (each voxel's sum
// is computed by one thread in tap order, so the result does not depend on the
// thread count).
#include <chrono>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <unordered_map>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

struct Site {
  int32_t b, x, y, z;
  bool operator==(const Site& o) const {
    return b == o.b && x == o.x && y == o.y && z == o.z;
  }
};

struct SiteHash {
  size_t operator()(const Site& s) const {
    // Two 64-bit halves, each holding two full int32 fields, mixed by std::hash.
    uint64_t lo = (uint64_t(uint32_t(s.b)) << 32) | uint32_t(s.x);
    uint64_t hi = (uint64_t(uint32_t(s.y)) << 32) | uint32_t(s.z);
    size_t h = std::hash<uint64_t>()(lo);
    return h ^ (std::hash<uint64_t>()(hi) + 0x9e3779b97f4a7c15ULL + (h << 6) + (h >> 2));
  }
};

double ms_since(std::chrono::steady_clock::time_point t0) {
  return std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
}

}  // namespace

extern "C" {

int oracle_num_threads() {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// Neighbour map.  coords: int32 [n, 4] = (b, x, y, z).  nbr_out: int32
// [n, K^3].  Returns 0, or -2 on a duplicate coordinate (nbr_out is then
// undefined), -1 on bad arguments.  ms_dict / ms_query (optional) receive the
// wall time of the dictionary build and of the lookups.
int oracle_neighbor_map(const int32_t* coords, int64_t n, int32_t K, int32_t stride,
                        int32_t* nbr_out, double* ms_dict, double* ms_query) {
  if (n < 0 || K < 1 || K % 2 == 0 || (n > 0 && (!coords || !nbr_out))) return -1;
  auto t0 = std::chrono::steady_clock::now();
  std::unordered_map<Site, int64_t, SiteHash> table;
  table.reserve(size_t(n) * 2 + 1);
  for (int64_t i = 0; i < n; ++i) {
    Site s{coords[4 * i + 0], coords[4 * i + 1], coords[4 * i + 2], coords[4 * i + 3]};
    if (!table.emplace(s, i).second) return -2;
  }
  if (ms_dict) *ms_dict = ms_since(t0);
  t0 = std::chrono::steady_clock::now();
  const int r = K / 2;
  const int64_t taps = int64_t(K) * K * K;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    const int32_t* c = coords + 4 * i;
    int64_t k = 0;
    for (int dx = -r; dx <= r; ++dx)
      for (int dy = -r; dy <= r; ++dy)
        for (int dz = -r; dz <= r; ++dz, ++k) {
          int64_t nx = int64_t(c[1]) + int64_t(stride) * dx;
          int64_t ny = int64_t(c[2]) + int64_t(stride) * dy;
          int64_t nz = int64_t(c[3]) + int64_t(stride) * dz;
          int32_t v = -1;
          if (nx >= INT32_MIN && nx <= INT32_MAX && ny >= INT32_MIN && ny <= INT32_MAX &&
              nz >= INT32_MIN && nz <= INT32_MAX) {
            auto it = table.find(Site{c[0], int32_t(nx), int32_t(ny), int32_t(nz)});
            if (it != table.end()) v = int32_t(it->second);
          }
          nbr_out[i * taps + k] = v;
        }
  }
  if (ms_query) *ms_query = ms_since(t0);
  return 0;
}

// Convolution for a list of output rows.  feats: double [n, cin]; W: double
// [taps, cin, cout]; nbr: int32 [n, taps]; rows: int64 [nrows] (the output
// rows to compute; nullptr means all n rows, in order).  out / scale: double
// [nrows, cout]; scale[r] = sum_k |feats[j]| @ |W[k]| (may be nullptr).
int oracle_submconv(const double* feats, const double* W, const int32_t* nbr, int64_t n,
                    int32_t taps, int32_t cin, int32_t cout, const int64_t* rows,
                    int64_t nrows, double* out, double* scale, double* ms_conv) {
  if (n < 0 || taps < 1 || cin < 1 || cout < 1 || nrows < 0) return -1;
  if (!rows) nrows = n;
  auto t0 = std::chrono::steady_clock::now();
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 64) reduction(| : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t i = rows ? rows[r] : r;
    double* acc = out + r * cout;
    double* mag = scale ? scale + r * cout : nullptr;
    for (int32_t co = 0; co < cout; ++co) acc[co] = 0.0;
    if (mag)
      for (int32_t co = 0; co < cout; ++co) mag[co] = 0.0;
    if (i < 0 || i >= n) {
      bad = 1;
      continue;
    }
    for (int32_t k = 0; k < taps; ++k) {
      int64_t j = nbr[i * taps + k];
      if (j < 0) continue;
      if (j >= n) {
        bad = 1;
        continue;
      }
      const double* f = feats + j * cin;
      const double* w = W + int64_t(k) * cin * cout;
      for (int32_t ci = 0; ci < cin; ++ci) {
        const double fv = f[ci];
        const double* wr = w + int64_t(ci) * cout;
        for (int32_t co = 0; co < cout; ++co) acc[co] += fv * wr[co];
        if (mag) {
          const double af = std::fabs(fv);
          for (int32_t co = 0; co < cout; ++co) mag[co] += af * std::fabs(wr[co]);
        }
      }
    }
  }
  if (ms_conv) *ms_conv = ms_since(t0);
  return bad ? -1 : 0;
}

// Input gradient (the adjoint of oracle_submconv in feats): every forward
// term feats[j] @ W[k] added to out[i] (j = nbr[i, k]) sends W[k] @ grad_out[i]
// back to row j.  The (i, k) pairs of each row j are listed first (i, then k,
// ascending), then every row j sums its own list, so the result does not
// depend on the thread count.  grad_out: double [n, cout]; gin / scale:
// double [n, cin]; scale (may be nullptr) is the same sum over |W| |grad_out|.
int oracle_submconv_backward_input(const double* grad_out, const double* W, const int32_t* nbr,
                                   int64_t n, int32_t taps, int32_t cin, int32_t cout,
                                   double* gin, double* scale, double* ms) {
  if (n < 0 || taps < 1 || cin < 1 || cout < 1) return -1;
  auto t0 = std::chrono::steady_clock::now();
  std::vector<int64_t> start(size_t(n) + 1, 0);
  for (int64_t i = 0; i < n * taps; ++i) {
    const int64_t j = nbr[i];
    if (j >= n) return -1;
    if (j >= 0) ++start[size_t(j) + 1];
  }
  for (int64_t j = 0; j < n; ++j) start[size_t(j) + 1] += start[size_t(j)];
  std::vector<int64_t> list(size_t(start[size_t(n)]));  // entries i * taps + k
  std::vector<int64_t> fill(start.begin(), start.end() - 1);
  for (int64_t e = 0; e < n * taps; ++e) {
    const int64_t j = nbr[e];
    if (j >= 0) list[size_t(fill[size_t(j)]++)] = e;
  }
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t j = 0; j < n; ++j) {
    double* acc = gin + j * cin;
    double* mag = scale ? scale + j * cin : nullptr;
    for (int32_t ci = 0; ci < cin; ++ci) acc[ci] = 0.0;
    if (mag)
      for (int32_t ci = 0; ci < cin; ++ci) mag[ci] = 0.0;
    for (int64_t e = start[size_t(j)]; e < start[size_t(j) + 1]; ++e) {
      const int64_t i = list[size_t(e)] / taps, k = list[size_t(e)] % taps;
      const double* g = grad_out + i * cout;
      const double* w = W + k * cin * cout;
      for (int32_t ci = 0; ci < cin; ++ci) {
        const double* wr = w + int64_t(ci) * cout;
        double s = 0.0, m = 0.0;
        for (int32_t co = 0; co < cout; ++co) {
          s += wr[co] * g[co];
          if (mag) m += std::fabs(wr[co]) * std::fabs(g[co]);
        }
        acc[ci] += s;
        if (mag) mag[ci] += m;
      }
    }
  }
  if (ms) *ms = ms_since(t0);
  return 0;
}

// Weight gradient (the adjoint of oracle_submconv in W): dW[k] is the sum
// over voxels i with a neighbour j = nbr[i, k] of outer(feats[j], grad_out[i]),
// voxels in ascending order.  feats: double [n, cin]; grad_out: double
// [n, cout]; dW / scale: double [taps, cin, cout] (scale may be nullptr).
int oracle_submconv_backward_weight(const double* feats, const double* grad_out,
                                    const int32_t* nbr, int64_t n, int32_t taps, int32_t cin,
                                    int32_t cout, double* dW, double* scale, double* ms) {
  if (n < 0 || taps < 1 || cin < 1 || cout < 1) return -1;
  auto t0 = std::chrono::steady_clock::now();
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t kc = 0; kc < int64_t(taps) * cin; ++kc) {
    const int64_t k = kc / cin, ci = kc % cin;
    double* acc = dW + kc * cout;
    double* mag = scale ? scale + kc * cout : nullptr;
    for (int32_t co = 0; co < cout; ++co) acc[co] = 0.0;
    if (mag)
      for (int32_t co = 0; co < cout; ++co) mag[co] = 0.0;
    for (int64_t i = 0; i < n; ++i) {
      const int64_t j = nbr[i * taps + k];
      if (j < 0) continue;
      if (j >= n) {
        bad = 1;
        continue;
      }
      const double fv = feats[j * cin + ci];
      const double* g = grad_out + i * cout;
      for (int32_t co = 0; co < cout; ++co) acc[co] += fv * g[co];
      if (mag) {
        const double af = std::fabs(fv);
        for (int32_t co = 0; co < cout; ++co) mag[co] += af * std::fabs(g[co]);
      }
    }
  }
  if (ms) *ms = ms_since(t0);
  return bad ? -1 : 0;
}

}  // extern "C"
