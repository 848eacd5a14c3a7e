/* A plain C99 program that drives the GPU path through the C ABI alone: device
 * buffers come from the CUDA runtime, nothing from Python.  Two problems whose
 * answers follow from the definition of the loss:
 *
 *   1. K = 1.  The teacher puts all its mass on one id per row, so the loss of
 *      a row is the student's cross-entropy at that id,
 *        l_r = LSE(z_r / T) - z_r[id_r] / T,
 *      averaged over the unmasked rows, and dlogits_r = (q_r - e_id) / (T N_v).
 *      The reference is computed here in double from the same bf16 inputs.
 *   2. K = V and the teacher's logits equal the student's own (computed here),
 *      so p = q: the loss and both gradients vanish.
 *
 * Prints one line per check; exit status 0 when all hold. */
#include <cuda_runtime_api.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "fckl.h"

static int failures = 0;
#define CHECK(cond, ...)                                       \
  do {                                                         \
    printf("%s ", (cond) ? "ok  " : "FAIL");                   \
    printf(__VA_ARGS__);                                       \
    printf("\n");                                              \
    if (!(cond)) ++failures;                                   \
  } while (0)

/* float -> bfloat16 bits, round to nearest even (inputs are finite) */
static uint16_t to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
static double from_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* xorshift64* and Box-Muller: seeded inputs, independent of any other generator */
static uint64_t rng_state = 0x9E3779B97F4A7C15ull;
static double uniform01(void) {
  rng_state ^= rng_state >> 12;
  rng_state ^= rng_state << 25;
  rng_state ^= rng_state >> 27;
  return (double)((rng_state * 0x2545F4914F6CDD1Dull) >> 11) * (1.0 / 9007199254740992.0);
}
static double normal(double sd) {
  const double u1 = uniform01() + 1e-300, u2 = uniform01();
  return sd * sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

#define CUDA_OK(x)                                                           \
  do {                                                                       \
    cudaError_t e_ = (x);                                                    \
    if (e_ != cudaSuccess) {                                                 \
      printf("FAIL %s: %s\n", #x, cudaGetErrorString(e_));                   \
      exit(2);                                                               \
    }                                                                        \
  } while (0)

typedef struct {
  int N, H, V, K;
  float T;
  int chunk;
  int mask_every;  /* mask row r when r % mask_every == 3 (0: no mask) */
  double w_sd;
  int self_teacher; /* 1: K = V, teacher logits = the student's logits */
} Case;

static double frob(const double* a, size_t n) {
  double s = 0;
  for (size_t i = 0; i < n; ++i) s += a[i] * a[i];
  return sqrt(s);
}

static void run_case(const char* name, const Case* c) {
  const int N = c->N, H = c->H, V = c->V, K = c->K;
  const double T = c->T;
  uint16_t* hb = malloc(sizeof(uint16_t) * N * H);
  uint16_t* wb = malloc(sizeof(uint16_t) * V * H);
  double* hd = malloc(sizeof(double) * N * H);
  double* wd = malloc(sizeof(double) * V * H);
  int32_t* ids = malloc(sizeof(int32_t) * N * K);
  float* lg = malloc(sizeof(float) * N * K);
  uint8_t* mask = malloc((size_t)N);
  double* z = malloc(sizeof(double) * N * V);
  double* g = calloc((size_t)N * V, sizeof(double));
  double* dH_ref = calloc((size_t)N * H, sizeof(double));
  double* dW_ref = calloc((size_t)V * H, sizeof(double));
  float* dH = malloc(sizeof(float) * N * H);
  float* dW = malloc(sizeof(float) * V * H);
  double* diff = malloc(sizeof(double) * (N > V ? N : V) * H);
  int r, v, k, j;

  for (r = 0; r < N * H; ++r) { hb[r] = to_bf16((float)normal(1.0)); hd[r] = from_bf16(hb[r]); }
  for (r = 0; r < V * H; ++r) { wb[r] = to_bf16((float)normal(c->w_sd)); wd[r] = from_bf16(wb[r]); }
  for (r = 0; r < N; ++r) mask[r] = (uint8_t)(c->mask_every && r % c->mask_every == 3 ? 0 : 1);
  for (r = 0; r < N; ++r)
    for (v = 0; v < V; ++v) {
      double s = 0;
      for (j = 0; j < H; ++j) s += hd[(size_t)r * H + j] * wd[(size_t)v * H + j];
      z[(size_t)r * V + v] = s;
    }
  for (r = 0; r < N; ++r) {
    if (c->self_teacher) {  /* a random permutation of the vocabulary, z at each id */
      for (k = 0; k < K; ++k) ids[(size_t)r * K + k] = k;
      for (k = K - 1; k > 0; --k) {
        const int i = (int)(uniform01() * (k + 1));
        const int32_t t = ids[(size_t)r * K + k];
        ids[(size_t)r * K + k] = ids[(size_t)r * K + i];
        ids[(size_t)r * K + i] = t;
      }
      for (k = 0; k < K; ++k) lg[(size_t)r * K + k] = (float)z[(size_t)r * V + ids[(size_t)r * K + k]];
    } else {
      for (k = 0; k < K; ++k) {
        ids[(size_t)r * K + k] = (int32_t)(uniform01() * V);
        lg[(size_t)r * K + k] = (float)normal(3.0);
      }
    }
  }

  /* reference (case 1; for case 2 the answer is 0) */
  int nv = 0;
  for (r = 0; r < N; ++r) nv += mask[r] != 0;
  double loss_ref = 0;
  if (!c->self_teacher) {
    for (r = 0; r < N; ++r) {
      if (!mask[r]) continue;
      const double* zr = z + (size_t)r * V;
      double m = -INFINITY, s = 0;
      for (v = 0; v < V; ++v) m = fmax(m, zr[v] / T);
      for (v = 0; v < V; ++v) s += exp(zr[v] / T - m);
      const double lse = m + log(s);
      const int id = ids[(size_t)r * K];
      loss_ref += lse - zr[id] / T;
      for (v = 0; v < V; ++v) g[(size_t)r * V + v] = exp(zr[v] / T - lse) / (T * nv);
      g[(size_t)r * V + id] -= 1.0 / (T * nv);
    }
    loss_ref /= nv;
    for (r = 0; r < N; ++r)
      for (v = 0; v < V; ++v) {
        const double gv = g[(size_t)r * V + v];
        if (gv == 0) continue;
        for (j = 0; j < H; ++j) {
          dH_ref[(size_t)r * H + j] += gv * wd[(size_t)v * H + j];
          dW_ref[(size_t)v * H + j] += gv * hd[(size_t)r * H + j];
        }
      }
  }

  /* the library, through its C ABI, on device buffers */
  fckl_problem p;
  memset(&p, 0, sizeof p);
  p.N = N; p.H = H; p.V = V; p.K = K; p.T = c->T; p.chunk = c->chunk;
  p.teacher = FCKL_TEACHER_LOGITS;
  const size_t ws_bytes = fckl_workspace_bytes(&p);
  void *d_h, *d_w, *d_ids, *d_lg, *d_mask, *d_loss, *d_dH, *d_dW, *d_ws;
  CUDA_OK(cudaMalloc(&d_h, sizeof(uint16_t) * N * H));
  CUDA_OK(cudaMalloc(&d_w, sizeof(uint16_t) * V * H));
  CUDA_OK(cudaMalloc(&d_ids, sizeof(int32_t) * N * K));
  CUDA_OK(cudaMalloc(&d_lg, sizeof(float) * N * K));
  CUDA_OK(cudaMalloc(&d_mask, (size_t)N));
  CUDA_OK(cudaMalloc(&d_loss, sizeof(float)));
  CUDA_OK(cudaMalloc(&d_dH, sizeof(float) * N * H));
  CUDA_OK(cudaMalloc(&d_dW, sizeof(float) * V * H));
  CUDA_OK(cudaMalloc(&d_ws, ws_bytes));
  CUDA_OK(cudaMemcpy(d_h, hb, sizeof(uint16_t) * N * H, cudaMemcpyHostToDevice));
  CUDA_OK(cudaMemcpy(d_w, wb, sizeof(uint16_t) * V * H, cudaMemcpyHostToDevice));
  CUDA_OK(cudaMemcpy(d_ids, ids, sizeof(int32_t) * N * K, cudaMemcpyHostToDevice));
  CUDA_OK(cudaMemcpy(d_lg, lg, sizeof(float) * N * K, cudaMemcpyHostToDevice));
  CUDA_OK(cudaMemcpy(d_mask, mask, (size_t)N, cudaMemcpyHostToDevice));

  fckl_status st = fckl_fwd_bwd(&p, d_h, d_w, d_ids, d_lg, c->mask_every ? d_mask : NULL,
                                d_loss, NULL, d_dH, d_dW, d_ws, ws_bytes, NULL);
  CHECK(st == FCKL_OK, "%s: fckl_fwd_bwd -> %s", name, fckl_status_string(st));
  st = fckl_check(d_ws, NULL);
  CHECK(st == FCKL_OK, "%s: fckl_check -> %s", name, fckl_status_string(st));
  float loss = 0;
  CUDA_OK(cudaMemcpy(&loss, d_loss, sizeof(float), cudaMemcpyDeviceToHost));
  CUDA_OK(cudaMemcpy(dH, d_dH, sizeof(float) * N * H, cudaMemcpyDeviceToHost));
  CUDA_OK(cudaMemcpy(dW, d_dW, sizeof(float) * V * H, cudaMemcpyDeviceToHost));

  if (!c->self_teacher) {
    const double rel_loss = fabs(loss - loss_ref) / fabs(loss_ref);
    CHECK(rel_loss <= 1e-3, "%s: loss %.7f vs %.7f (rel %.2e, N_v %d)", name, loss, loss_ref,
          rel_loss, nv);
    for (r = 0; r < N * H; ++r) diff[r] = dH[r] - dH_ref[r];
    const double eh = frob(diff, (size_t)N * H) / frob(dH_ref, (size_t)N * H);
    CHECK(eh <= 2e-2, "%s: dH rel Frobenius %.2e", name, eh);
    for (r = 0; r < V * H; ++r) diff[r] = dW[r] - dW_ref[r];
    const double ew = frob(diff, (size_t)V * H) / frob(dW_ref, (size_t)V * H);
    CHECK(ew <= 2e-2, "%s: dW rel Frobenius %.2e", name, ew);
    int masked_zero = 1;
    for (r = 0; r < N; ++r)
      if (!mask[r])
        for (j = 0; j < H; ++j) masked_zero &= dH[(size_t)r * H + j] == 0.0f;
    CHECK(masked_zero, "%s: dH rows of masked rows are zero", name);
  } else {
    double mh = 0, mw = 0;
    for (r = 0; r < N * H; ++r) mh = fmax(mh, fabs(dH[r]));
    for (r = 0; r < V * H; ++r) mw = fmax(mw, fabs(dW[r]));
    CHECK(fabs(loss) <= 5e-5, "%s: loss %.3e (teacher = student)", name, loss);
    /* a teacher that differs gives entries of order 1/(T N_v) * |W| ~ 1e-2 here */
    CHECK(mh <= 1e-5 && mw <= 1e-5, "%s: max |dH| %.2e, max |dW| %.2e", name, mh, mw);
  }

  cudaFree(d_h); cudaFree(d_w); cudaFree(d_ids); cudaFree(d_lg); cudaFree(d_mask);
  cudaFree(d_loss); cudaFree(d_dH); cudaFree(d_dW); cudaFree(d_ws);
  free(hb); free(wb); free(hd); free(wd); free(ids); free(lg); free(mask); free(z); free(g);
  free(dH_ref); free(dW_ref); free(dH); free(dW); free(diff);
}

int main(void) {
  /* ragged rows (130 over chunks of 64), H % 64 != 0, a padded last vocabulary tile */
  const Case ce = {130, 72, 1000, 1, 1.5f, 64, 7, 0.05, 0};
  /* K = V = 200, the teacher's logits are the student's own */
  const Case self = {96, 64, 200, 200, 0.8f, 0, 0, 0.5, 1};
  run_case("cross-entropy (K = 1)", &ce);
  run_case("teacher = student (K = V)", &self);
  printf("%d failure(s)\n", failures);
  return failures == 0 ? 0 : 1;
}
