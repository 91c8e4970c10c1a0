// Internal host-side launchers behind the C ABI (not exported).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "lrkv.h"

namespace lrkv {

// SM count and opt-in shared memory per block of a device.
struct DevInfo {
  int sms, optin;
};
// The current device and its DevInfo, queried once per device per process.
int current_device_info(int& dev, DevInfo& info);
// Once per (kernel, device): allow the device's full opt-in dynamic shared
// memory for fn and, when max_carveout, prefer the largest shared-memory
// carveout.  Later calls return at once.
int prepare_kernel(const void* fn, bool max_carveout);

// Launch fn as the programmatic dependent of the stream's previous kernel
// (it may start before that grid ends and waits for it with
// griddepcontrol.wait before reading what that grid writes).
cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       void** args);

struct DecodeLaunch {
  int B, H_kv, H_q, dtype;
  const int* seq_len;
  int n_sink, W;
  const void* codes;  // latent slabs (nullptr: no latent space)
  const int* bt_lat;
  int maxp_lat, rk, rv, num_pages_lat;
  const void* fr;     // full-rank tiles (nullptr: no full-rank space)
  const int* bt_fr;
  int maxp_fr, num_pages_fr;
  const void* q;
  const float *P_k, *P_v;
  long long basis_bs;
  float scale;
  void* o;
  void* ws;
  size_t ws_bytes;
  const float* A = nullptr;  // value predictors of a value-amortised cache
};

size_t decode_workspace_bytes(int B, int H_kv, int H_q, int rk, int rv, bool has_lat,
                              bool has_fr, int dtype);
// Status of planning that decode (LRKV_OK when decode_workspace_bytes > 0).
int decode_plan_check(int B, int H_kv, int H_q, int rk, int rv, bool has_lat, bool has_fr,
                      int dtype);
// Status explaining a zero lrkv_decode_workspace_bytes for this cache.
int decode_plan_status(const lrkv_cache* cache, int H_q);
// The query fold of a decode step, done by the append kernel: q (cache
// dtype, [B][H_q][128]) -> qlat [B][H_q][rk] = qscale P_k^T q and, when qfr
// is set, qfr [B][H_q][128] = qscale q (qscale = scale log2 e).
struct StepFold {
  const void* q;
  int H_q;
  float qscale;
  float *qlat, *qfr;
};
// folded == true: a decode step whose queries the append kernel just folded
// into the workspace (decode_fold_targets); the q-fold launch is skipped and
// the split kernel waits for the append before reading the cache.
int decode_launch(const DecodeLaunch& L, cudaStream_t st, bool folded = false);
// Workspace addresses the q-fold of L writes (qfr == nullptr: no full-rank
// space); a status other than LRKV_OK when L cannot be planned.
int decode_fold_targets(const DecodeLaunch& L, float** qlat, float** qfr, float* qscale);

int compress_launch(const lrkv_cache& c, const void* k, const void* v, int n, const int* n_new,
                    long long seq_stride, long long head_stride, const float* P_k,
                    const float* P_v, long long basis_bs, cudaStream_t st,
                    const float* A = nullptr, const StepFold* fold = nullptr);
int dense_append_launch(const lrkv_dense_cache& c, const void* k, const void* v, int n,
                        const int* n_new,
                        long long seq_stride, long long head_stride, cudaStream_t st);

int oja_launch(float* P, int S, int r, long long basis_stride, const void* x, int x_dtype,
               long long x_stride, int n, float eta, int qr_every, long long tokens_seen,
               cudaStream_t st);
int qr_launch(float* P, int S, int r, long long basis_stride, cudaStream_t st);
int oja_blocked_launch(float* P, int S, int r, long long basis_stride, const void* x,
                       int x_dtype, long long x_stride, int n, float eta, int qr_every,
                       long long tokens_seen, int chunk, cudaStream_t st);

size_t amortise_workspace_bytes(int B, int H_kv, int rk, int rv);
int amortise_launch(const lrkv_cache& c, const void* v, int n, long long seq_stride,
                    long long head_stride, const float* P_v, long long basis_bs, float* A,
                    void* ws, cudaStream_t st);

size_t rebase_workspace_bytes(int B, int H_kv, int rk, int rv);
int rebase_launch(const lrkv_cache& c, const float* Pk_old, const float* Pk_new,
                  const float* Pv_old, const float* Pv_new, long long basis_bs, void* ws,
                  cudaStream_t st);

}  // namespace lrkv
