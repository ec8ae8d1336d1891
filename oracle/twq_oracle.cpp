// TEST INFRASTRUCTURE ONLY. This oracle checks the CUDA path; nothing on the
// product path may link, load or call it. Only tests/, the smoke check and the
// benchmark's CPU-baseline leg use it.
//
// A plain, single-threaded CPU statement of the fused dual-component W4A4 +
// low-rank linear layer of TwinQuant ("TwinQuant: Learnable Subspace
// Decomposition for 4-Bit LLM Quantization", ICML'26):
//
//   Y = Q(X)*Q(R) + bf16( Q(X)*Q(L1) ) * L2        X in R^{b x m}, W = L1*L2 + R
//
// * Symmetric quantizer, Eq. (1) of §2 (blog digest): Q_X = round(X / s_X),
//   s_X = max|X| / q_max, q_max = 2^(k-1) - 1 = 7 for k = 4 bits.
// * Group-wise quantization with groups of 128 along the reduction dimension
//   for weights and activations, §5.1 (both the blog digest and the arXiv
//   summary).
// * Quantized linear layer, Eq. (2) of §2: XW ~ s_X s_W Q_X Q_W, applied per
//   group, so the integer dot product of each group is exact.
// * Dual-component form, Eq. (3) of §2, with the low-rank factor pair (U, V)
//   named (L1, L2) here; the learned transforms of §4.1 are already folded in.
// * Kernel dataflow, §4.3: one activation quantization reused by the residual
//   GEMM and the first low-rank GEMM; the first stage's result H is
//   converted and fed to the second stage; a single epilogue adds both parts.
//   Here the second stage takes H rounded to BF16 and L2 in BF16
//   (the page's on-the-fly INT4 requantization is composed from these functions
//   in oracle.layer_s2q), and Y is BF16.
//
// Written for readability, not speed. All products are accumulated in int64
// (group dot products) and double (scaled sums), in ascending group order.
// Compile with -O2 -fno-fast-math -ffp-contract=off on x86-64 (SSE2 floats).
#include <cmath>
#include <cstdint>
#include <cstring>

namespace {

constexpr int kGroup = 128;  // §5.1: group size 128
constexpr int kBits = 4;
constexpr int kQmax = (1 << (kBits - 1)) - 1;  // Eq. (1): q_max = 2^(k-1) - 1 = 7
// W4A8 (§5.1, the quantization settings: 4-bit weights, 8-bit activations):
// the same Eq. (1) with k = 8 for the activations, q_max = 127.
constexpr int kQmaxA8 = (1 << (8 - 1)) - 1;

float bf16_to_f32(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Round a float to BF16, nearest even (NaN -> canonical quiet NaN).
uint16_t f32_to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return static_cast<uint16_t>(u >> 16);
}

// Eq. (1) on one group: s = max|v| / q_max (one correctly rounded float
// division), q = clamp(round_half_even(v / s), -q_max, q_max) with a correctly
// rounded float division per element. An all-zero group has s = 0 and q = 0
// (Eq. (1) is 0/0 there).
void quantize_group(const float* v, int64_t stride, int count, int8_t* q, int64_t qstride,
                    float* s_out, int qmax = kQmax) {
  float a = 0.0f;
  for (int k = 0; k < count; ++k) {
    float m = std::fabs(v[k * stride]);
    if (m > a) a = m;
  }
  float s = a / static_cast<float>(qmax);
  *s_out = s;
  for (int k = 0; k < count; ++k) {
    int code = 0;
    if (s != 0.0f) {
      float t = v[k * stride] / s;
      float rounded = std::nearbyint(t);  // default rounding mode: half to even
      if (rounded > qmax) rounded = static_cast<float>(qmax);
      if (rounded < -qmax) rounded = static_cast<float>(-qmax);
      code = static_cast<int>(rounded);
    }
    q[k * qstride] = static_cast<int8_t>(code);
  }
}

}  // namespace

extern "C" {

int twq_ref_qmax() { return kQmax; }
int twq_ref_group() { return kGroup; }

// Eq. (1) on one group of float inputs (used by the pins on values that BF16
// cannot hold, e.g. float subnormals where the clamp matters).
int twq_ref_quant_group_f32(const float* v, int count, int8_t* q, float* s) {
  if (!v || !q || !s || count <= 0) return 1;
  quantize_group(v, 1, count, q, 1, s);
  return 0;
}

int twq_ref_qmax_a8() { return kQmaxA8; }

// Activation codes: X is rows x m BF16 (row stride ldx elements); groups of 128
// run along m within each row (one scale per token and group). qmax is 7 (W4A4)
// or 127 (the W4A8 activations).
// q: rows x m codes (row-major), s: rows x (m/128) scales (row-major).
int twq_ref_quantize_rows_q(const uint16_t* x, int64_t rows, int64_t m, int64_t ldx, int qmax,
                            int8_t* q, float* s) {
  if (!x || !q || !s || rows < 0 || m <= 0 || m % kGroup || ldx < m) return 1;
  if (qmax != kQmax && qmax != kQmaxA8) return 1;
  const int64_t G = m / kGroup;
  float buf[kGroup];
  for (int64_t i = 0; i < rows; ++i)
    for (int64_t g = 0; g < G; ++g) {
      for (int k = 0; k < kGroup; ++k) buf[k] = bf16_to_f32(x[i * ldx + g * kGroup + k]);
      quantize_group(buf, 1, kGroup, q + i * m + g * kGroup, 1, s + i * G + g, qmax);
    }
  return 0;
}

int twq_ref_quantize_rows(const uint16_t* x, int64_t rows, int64_t m, int64_t ldx, int8_t* q,
                          float* s) {
  return twq_ref_quantize_rows_q(x, rows, m, ldx, kQmax, q, s);
}

// Eq. (1) with q_max = 127 on one group of float inputs (pins on values BF16
// cannot hold).
int twq_ref_quant_group_f32_a8(const float* v, int count, int8_t* q, float* s) {
  if (!v || !q || !s || count <= 0) return 1;
  quantize_group(v, 1, count, q, 1, s, kQmaxA8);
  return 0;
}

// Weight codes: W is m x cols BF16 row-major; groups of 128 run along m within
// each column (one scale per output column and group).
// q: cols x m codes (column j's codes contiguous along k), s: (m/128) x cols.
int twq_ref_quantize_cols(const uint16_t* w, int64_t m, int64_t cols, int8_t* q, float* s) {
  if (!w || !q || !s || m <= 0 || m % kGroup || cols < 0) return 1;
  const int64_t G = m / kGroup;
  float buf[kGroup];
  for (int64_t j = 0; j < cols; ++j)
    for (int64_t g = 0; g < G; ++g) {
      for (int k = 0; k < kGroup; ++k) buf[k] = bf16_to_f32(w[(g * kGroup + k) * cols + j]);
      quantize_group(buf, 1, kGroup, q + j * m + g * kGroup, 1, s + g * cols + j);
    }
  return 0;
}

// Two's-complement nibbles, element 2p in the low nibble of byte p.
int twq_ref_pack_nibbles(const int8_t* q, int64_t count, uint8_t* out) {
  if (!q || !out || count % 2) return 1;
  for (int64_t p = 0; p < count / 2; ++p) {
    unsigned lo = static_cast<unsigned>(q[2 * p]) & 0xFu;
    unsigned hi = static_cast<unsigned>(q[2 * p + 1]) & 0xFu;
    out[p] = static_cast<uint8_t>(lo | (hi << 4));
  }
  return 0;
}

int twq_ref_unpack_nibbles(const uint8_t* in, int64_t count, int8_t* q) {
  if (!in || !q || count % 2) return 1;
  for (int64_t p = 0; p < count / 2; ++p) {
    int lo = in[p] & 0xF;
    int hi = (in[p] >> 4) & 0xF;
    q[2 * p] = static_cast<int8_t>(lo >= 8 ? lo - 16 : lo);
    q[2 * p + 1] = static_cast<int8_t>(hi >= 8 ? hi - 16 : hi);
  }
  return 0;
}

// The library's activation format: xq rows x (m/2) packed bytes, sx rows x (m/128).
int twq_ref_quantize_act(const uint16_t* x, int64_t rows, int64_t m, int64_t ldx, uint8_t* xq,
                         float* sx) {
  if (!xq) return 1;
  int8_t* q = new int8_t[rows * m > 0 ? rows * m : 1];
  int rc = twq_ref_quantize_rows(x, rows, m, ldx, q, sx);
  if (rc == 0) rc = twq_ref_pack_nibbles(q, rows * m, xq);
  delete[] q;
  return rc;
}

// The library's weight format.
//   rq  : n x (m/2) packed codes of R, column j contiguous along k
//   sr  : (m/128) x n scales of R
//   l1q : r x (m/2) packed codes of L1
//   sl1 : (m/128) x r scales of L1
//   l2t : n x r BF16, the transpose of L2 (unquantized)
int twq_ref_pack_weights(const uint16_t* R, const uint16_t* L1, const uint16_t* L2, int64_t m,
                         int64_t n, int64_t r, uint8_t* rq, float* sr, uint8_t* l1q, float* sl1,
                         uint16_t* l2t) {
  if (m <= 0 || m % kGroup || n <= 0 || r < 0) return 1;
  int8_t* q = new int8_t[n * m];
  int rc = twq_ref_quantize_cols(R, m, n, q, sr);
  if (rc == 0) rc = twq_ref_pack_nibbles(q, n * m, rq);
  delete[] q;
  if (rc || r == 0) return rc;
  q = new int8_t[r * m];
  rc = twq_ref_quantize_cols(L1, m, r, q, sl1);
  if (rc == 0) rc = twq_ref_pack_nibbles(q, r * m, l1q);
  delete[] q;
  if (rc) return rc;
  for (int64_t c = 0; c < r; ++c)
    for (int64_t j = 0; j < n; ++j) l2t[j * r + c] = L2[c * n + j];
  return 0;
}

// Modes of twq_ref_linear.
enum { TWQ_REF_FUSED = 0, TWQ_REF_W4A4_ONLY = 1, TWQ_REF_LOWRANK_ONLY = 2 };

// The layer on unpacked codes, for the rows listed in `rows` (all rows if
// rows == NULL; then nrows == b). Outputs are nrows x n (y, y64) and
// nrows x r (h64, hb), any of which may be NULL.
//
//   I_g[i,j]   = sum_{k in g} qx[i,k] * qr[j,k]                (int64, exact)
//   Yres[i,j]  = sum_g sx[i,g] * sr[g,j] * I_g[i,j]            (double, ascending g)
//   H[i,c]     = sum_g sx[i,g] * sl1[g,c] * sum_{k in g} qx[i,k] * ql1[c,k]
//   Hb[i,c]    = bf16(float(H[i,c]))
//   Ylr[i,j]   = sum_c Hb[i,c] * L2[c,j]                       (double, ascending c)
//   Y[i,j]     = bf16(float(Yres + Ylr))
// TWQ_REF_W4A4_ONLY drops Ylr; TWQ_REF_LOWRANK_ONLY drops Yres.
int twq_ref_linear(const int8_t* qx, const float* sx, int64_t b, int64_t m, const int8_t* qr,
                   const float* sr, int64_t n, const int8_t* ql1, const float* sl1, int64_t r,
                   const uint16_t* l2, int mode, const int64_t* rows, int64_t nrows, uint16_t* y,
                   double* y64, double* h64, uint16_t* hb_out) {
  if (!qx || !sx || m <= 0 || m % kGroup || n <= 0 || r < 0 || b < 0) return 1;
  if (mode < 0 || mode > 2) return 1;
  const bool use_res = mode != TWQ_REF_LOWRANK_ONLY;
  const bool use_lr = mode != TWQ_REF_W4A4_ONLY && r > 0;
  if (use_res && (!qr || !sr)) return 1;
  if (use_lr && (!ql1 || !sl1 || !l2)) return 1;
  if (!rows) nrows = b;
  const int64_t G = m / kGroup;
  double* yres = new double[n];
  double* h = new double[r > 0 ? r : 1];
  double* hb = new double[r > 0 ? r : 1];
  for (int64_t t = 0; t < nrows; ++t) {
    const int64_t i = rows ? rows[t] : t;
    if (i < 0 || i >= b) {
      delete[] yres;
      delete[] h;
      delete[] hb;
      return 1;
    }
    const int8_t* xi = qx + i * m;
    for (int64_t j = 0; j < n; ++j) yres[j] = 0.0;
    if (use_res) {
      for (int64_t j = 0; j < n; ++j) {
        const int8_t* wj = qr + j * m;
        double acc = 0.0;
        for (int64_t g = 0; g < G; ++g) {
          int64_t dot = 0;
          for (int k = 0; k < kGroup; ++k)
            dot += static_cast<int64_t>(xi[g * kGroup + k]) * wj[g * kGroup + k];
          acc += static_cast<double>(sx[i * G + g]) * static_cast<double>(sr[g * n + j]) *
                 static_cast<double>(dot);
        }
        yres[j] = acc;
      }
    }
    if (use_lr) {
      for (int64_t c = 0; c < r; ++c) {
        const int8_t* lc = ql1 + c * m;
        double acc = 0.0;
        for (int64_t g = 0; g < G; ++g) {
          int64_t dot = 0;
          for (int k = 0; k < kGroup; ++k)
            dot += static_cast<int64_t>(xi[g * kGroup + k]) * lc[g * kGroup + k];
          acc += static_cast<double>(sx[i * G + g]) * static_cast<double>(sl1[g * r + c]) *
                 static_cast<double>(dot);
        }
        h[c] = acc;
        uint16_t hbits = f32_to_bf16(static_cast<float>(acc));
        hb[c] = static_cast<double>(bf16_to_f32(hbits));
        if (h64) h64[t * r + c] = acc;
        if (hb_out) hb_out[t * r + c] = hbits;
      }
    }
    for (int64_t j = 0; j < n; ++j) {
      double ylr = 0.0;
      if (use_lr)
        for (int64_t c = 0; c < r; ++c) ylr += hb[c] * static_cast<double>(bf16_to_f32(l2[c * n + j]));
      double total = use_res ? yres[j] + ylr : ylr;
      if (y64) y64[t * n + j] = total;
      if (y) y[t * n + j] = f32_to_bf16(static_cast<float>(total));
    }
  }
  delete[] yres;
  delete[] h;
  delete[] hb;
  return 0;
}

// Brute force for the pins: dequantize first (s * q, Eq. (1)'s Q(X) = s_X Q_X),
// then multiply in double with no grouping. Same output convention as
// twq_ref_linear (y64 only, all rows).
int twq_ref_dequant_matmul(const int8_t* qx, const float* sx, int64_t b, int64_t m,
                           const int8_t* qr, const float* sr, int64_t n, const int8_t* ql1,
                           const float* sl1, int64_t r, const uint16_t* l2, int mode,
                           double* y64) {
  if (!qx || !sx || !y64 || m <= 0 || m % kGroup) return 1;
  const bool use_res = mode != TWQ_REF_LOWRANK_ONLY;
  const bool use_lr = mode != TWQ_REF_W4A4_ONLY && r > 0;
  const int64_t G = m / kGroup;
  double* xd = new double[m];
  double* hb = new double[r > 0 ? r : 1];
  for (int64_t i = 0; i < b; ++i) {
    for (int64_t k = 0; k < m; ++k)
      xd[k] = static_cast<double>(sx[i * G + k / kGroup]) * qx[i * m + k];
    if (use_lr)
      for (int64_t c = 0; c < r; ++c) {
        double acc = 0.0;
        for (int64_t k = 0; k < m; ++k)
          acc += xd[k] * (static_cast<double>(sl1[(k / kGroup) * r + c]) * ql1[c * m + k]);
        hb[c] = static_cast<double>(bf16_to_f32(f32_to_bf16(static_cast<float>(acc))));
      }
    for (int64_t j = 0; j < n; ++j) {
      double acc = 0.0;
      if (use_res)
        for (int64_t k = 0; k < m; ++k)
          acc += xd[k] * (static_cast<double>(sr[(k / kGroup) * n + j]) * qr[j * m + k]);
      if (use_lr)
        for (int64_t c = 0; c < r; ++c) acc += hb[c] * static_cast<double>(bf16_to_f32(l2[c * n + j]));
      y64[i * n + j] = acc;
    }
  }
  delete[] xd;
  delete[] hb;
  return 0;
}

uint16_t twq_ref_f32_to_bf16(float f) { return f32_to_bf16(f); }

}  // extern "C"
