// extern "C" entry points of libkronq (declared in include/kronq.h).
// Host-side argument checks live next to each launcher; this file only maps
// the ABI onto them and provides the shared host helpers.
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"

size_t kq_cholesky_ws(int64_t n);
size_t kq_biip_ws(int64_t m, int64_t n);
size_t kq_quantize_ws(int64_t m, int64_t n);
size_t kq_loss_ws(int64_t m, int64_t n);
int kq_covariance(const uint16_t* A, int64_t N, int64_t d, int64_t lda, float* H, int64_t ldh,
                  float alpha, float beta, int32_t* info, cudaStream_t st);
int kq_sensitivity(const float* HX, int64_t n, const float* HG, int64_t m, double* out,
                   cudaStream_t st);
int kq_biip_rotate(float* W, int64_t m, int64_t n, float* HX, float* HG, const int8_t* su,
                   const int8_t* sv, float alpha, int mode, int inverse, float* SX, float* SG,
                   void* ws, size_t ws_bytes, cudaStream_t st);
int kq_cholesky_inv(const float* H, int64_t n, float damp_rel, float* U, int32_t* info, void* ws,
                    size_t ws_bytes, cudaStream_t st);
int kq_quantize_layer(float* W, int64_t m, int64_t n, const float* U, int bits, int group,
                      int block, int options, uint8_t* codes, float* scales, uint8_t* zeros,
                      float* W_hat, int32_t* info, void* ws, size_t ws_bytes, cudaStream_t st);
int kq_act_order(const float* H, int64_t n, int32_t* perm, cudaStream_t st);
size_t kq_deploy_ws(int64_t m, int64_t n, int64_t batch);
int kq_deploy_matvec(const uint32_t* packed, int64_t m, int64_t n, int bits, int group,
                     const float* scales, const uint8_t* zeros, const float* SX, const float* SG,
                     const int8_t* su, const int8_t* sv, int mode, const float* x, int64_t batch,
                     float* y, void* ws, size_t ws_bytes, cudaStream_t st);
int kq_permute(const void* src, void* dst, int64_t m, int64_t n, int elem_bytes,
               const int32_t* perm, int mode, int32_t* info, cudaStream_t st);
int kq_quantize_layer_noalloc(float* W, int64_t m, int64_t n, const float* U, int bits, int group,
                              int block, uint8_t* codes, float* scales, uint8_t* zeros,
                              float* W_hat, int32_t* info, cudaStream_t st);
int kq_pack(const uint8_t* codes, int64_t m, int64_t n, int bits, uint32_t* packed,
            cudaStream_t st);
size_t kq_drift_ws(int64_t n);
size_t kq_correction_ws(int64_t n);
size_t kq_quantize_asym_ws(int64_t m, int64_t n);
int kq_drift_covariance(const uint16_t* XqX, int64_t N, int64_t n, int64_t ld, float* H, float* A,
                        int32_t* info, void* ws, size_t ws_bytes, cudaStream_t st);
int kq_biip_rotate_input(float* A, int64_t n, const float* SX, const int8_t* sv, int mode,
                         void* ws, size_t ws_bytes, cudaStream_t st);
int kq_gptaq_correction(const float* A, const float* U, int64_t n, float alpha, float* P,
                        int32_t* info, void* ws, size_t ws_bytes, cudaStream_t st);
int kq_quantize_layer_asym(float* W, int64_t m, int64_t n, const float* U, const float* P,
                           int bits, int group, int block, uint8_t* codes, float* scales,
                           uint8_t* zeros, float* W_hat, int32_t* info, void* ws, size_t ws_bytes,
                           cudaStream_t st);
int kq_unpack(const uint32_t* packed, int64_t m, int64_t n, int bits, uint8_t* codes,
              cudaStream_t st);
int kq_layer_loss(const float* Wr, const float* Wh, int64_t m, int64_t n, const float* HX,
                  const float* HG, double* out, void* ws, size_t ws_bytes, cudaStream_t st);

namespace kqh {

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static std::atomic<unsigned long long> g_launches{0};

int launch_status() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? KRONQ_OK : KRONQ_ERR_CUDA;
}

unsigned long long launches() { return g_launches.load(std::memory_order_relaxed); }

// ---- launch timing: event pairs per device, reused after every enable
namespace {
struct TimerSlot {
  cudaEvent_t start, end;
  int category;
};
std::mutex g_timer_mu;
std::atomic<bool> g_timer_on{false};
std::vector<TimerSlot> g_timer_slots[64];
size_t g_timer_used[64] = {};
}  // namespace

int timer_begin(int category, cudaStream_t st) {
  if (!g_timer_on.load(std::memory_order_relaxed)) return -1;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  std::lock_guard<std::mutex> lock(g_timer_mu);
  std::vector<TimerSlot>& slots = g_timer_slots[dev];
  if (g_timer_used[dev] == slots.size()) {
    TimerSlot t;
    if (cudaEventCreate(&t.start) != cudaSuccess) return -1;
    if (cudaEventCreate(&t.end) != cudaSuccess) {
      cudaEventDestroy(t.start);
      return -1;
    }
    slots.push_back(t);
  }
  const size_t i = g_timer_used[dev]++;
  slots[i].category = category;
  if (cudaEventRecord(slots[i].start, st) != cudaSuccess) return -1;
  return dev * (1 << 24) + (int)i;
}

void timer_end(int slot, cudaStream_t st) {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lock(g_timer_mu);
  const int dev = slot >> 24;
  const size_t i = (size_t)(slot & ((1 << 24) - 1));
  if (dev < 64 && i < g_timer_used[dev]) cudaEventRecord(g_timer_slots[dev][i].end, st);
}

}  // namespace kqh

static cudaStream_t S(void* s) { return static_cast<cudaStream_t>(s); }

// Waits on an mbarrier that nothing ever arrives on, with the given limit:
// the bounded-wait path of the pipelined kernels, made to run out on purpose.
__global__ void selftest_wait_kernel(int32_t* info, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    kq::mbar_init(&bar, 1);
    abort = 0;
    kq::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) kq::mbar_wait(&bar, 0, &abort, info, limit_ns);
  __syncthreads();
}

extern "C" {

const char* kronq_status_string(int st) {
  switch (st) {
    case KRONQ_OK: return "ok";
    case KRONQ_ERR_INVALID_ARG: return "invalid argument";
    case KRONQ_ERR_UNSUPPORTED: return "unsupported";
    case KRONQ_ERR_NOT_PD: return "matrix not positive definite";
    case KRONQ_ERR_CUDA: return "CUDA error";
    case KRONQ_ERR_TIMEOUT: return "device wait timed out";
    case KRONQ_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int kronq_abi_version(void) { return 101; }

uint64_t kronq_launch_count(void) { return kqh::launches(); }

int kronq_timing_enable(int on) {
  std::lock_guard<std::mutex> lock(kqh::g_timer_mu);
  for (int d = 0; d < 64; ++d) kqh::g_timer_used[d] = 0;
  kqh::g_timer_on.store(on != 0);
  return KRONQ_OK;
}

int kronq_timing_read(int category, double* total_ms, uint64_t* launches) {
  if (!total_ms || !launches || category < 0 || category >= KRONQ_TIMER_COUNT)
    return KRONQ_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return KRONQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(kqh::g_timer_mu);
  double ms = 0.0;
  uint64_t count = 0;
  for (size_t i = 0; i < kqh::g_timer_used[dev]; ++i) {
    const kqh::TimerSlot& t = kqh::g_timer_slots[dev][i];
    if (t.category != category) continue;
    if (cudaEventSynchronize(t.end) != cudaSuccess) return KRONQ_ERR_CUDA;
    float e = 0.f;
    if (cudaEventElapsedTime(&e, t.start, t.end) != cudaSuccess) return KRONQ_ERR_CUDA;
    ms += e;
    ++count;
  }
  *total_ms = ms;
  *launches = count;
  return KRONQ_OK;
}

int kronq_selftest_wait(int32_t* info, int64_t limit_ns, void* stream) {
  if (!info || limit_ns <= 0 || limit_ns > 2000000000ll) return KRONQ_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, S(stream)>>>(info, (unsigned long long)limit_ns);
  return kqh::launch_status();
}

int kronq_sync_status(void* stream, const int32_t* info) {
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) {
    cudaGetLastError();
    return KRONQ_ERR_CUDA;
  }
  if (!info) return KRONQ_OK;
  int32_t v = 0;
  if (cudaMemcpy(&v, info, sizeof(v), cudaMemcpyDefault) != cudaSuccess) {
    cudaGetLastError();
    return KRONQ_ERR_CUDA;
  }
  return v;
}

size_t kronq_workspace_size(int64_t m, int64_t n, int bits, int group, int block) {
  (void)bits; (void)group; (void)block;
  if (m <= 0 || n <= 0) return 0;
  size_t s = kq_biip_ws(m, n);
  const size_t c = kq_cholesky_ws(n), q = kq_quantize_ws(m, n), l = kq_loss_ws(m, n);
  if (c > s) s = c;
  if (q > s) s = q;
  if (l > s) s = l;
  return s;
}

int kronq_covariance(const uint16_t* A, int64_t N, int64_t d, int64_t lda, float* H, int64_t ldh,
                     float alpha, float beta, int32_t* info, void* stream) {
  return kq_covariance(A, N, d, lda, H, ldh, alpha, beta, info, S(stream));
}

int kronq_sensitivity(const float* H_X, int64_t n, const float* H_G, int64_t m, double* out,
                      void* stream) {
  return kq_sensitivity(H_X, n, H_G, m, out, S(stream));
}

int kronq_biip_rotate(float* W, int64_t m, int64_t n, float* H_X, float* H_G,
                      const int8_t* sign_u, const int8_t* sign_v, float alpha, int mode,
                      int inverse, float* S_X, float* S_G, void* ws, size_t ws_bytes,
                      void* stream) {
  return kq_biip_rotate(W, m, n, H_X, H_G, sign_u, sign_v, alpha, mode, inverse, S_X, S_G, ws,
                        ws_bytes, S(stream));
}

int kronq_cholesky_inv(const float* H, int64_t n, float damp_rel, float* U_c, int32_t* info,
                       void* ws, size_t ws_bytes, void* stream) {
  return kq_cholesky_inv(H, n, damp_rel, U_c, info, ws, ws_bytes, S(stream));
}

int kronq_quantize_layer(float* W, int64_t m, int64_t n, const float* U_c, int bits, int group,
                         int block, uint8_t* codes, float* scales, uint8_t* zeros, float* W_hat,
                         int32_t* info, void* ws, size_t ws_bytes, void* stream) {
  return kq_quantize_layer(W, m, n, U_c, bits, group, block, 0, codes, scales, zeros, W_hat, info,
                           ws, ws_bytes, S(stream));
}

int kronq_quantize_layer_opt(float* W, int64_t m, int64_t n, const float* U_c, int bits,
                             int group, int block, int options, uint8_t* codes, float* scales,
                             uint8_t* zeros, float* W_hat, int32_t* info, void* ws,
                             size_t ws_bytes, void* stream) {
  return kq_quantize_layer(W, m, n, U_c, bits, group, block, options, codes, scales, zeros, W_hat,
                           info, ws, ws_bytes, S(stream));
}

int kronq_act_order(const float* H, int64_t n, int32_t* perm, void* stream) {
  return kq_act_order(H, n, perm, S(stream));
}

int kronq_permute(const void* src, void* dst, int64_t m, int64_t n, int elem_bytes,
                  const int32_t* perm, int mode, int32_t* info, void* stream) {
  return kq_permute(src, dst, m, n, elem_bytes, perm, mode, info, S(stream));
}

size_t kronq_deploy_workspace_size(int64_t m, int64_t n, int64_t batch) {
  return kq_deploy_ws(m, n, batch);
}

int kronq_deploy_matvec(const uint32_t* packed, int64_t m, int64_t n, int bits, int group,
                        const float* scales, const uint8_t* zeros, const float* S_X,
                        const float* S_G, const int8_t* sign_u, const int8_t* sign_v, int mode,
                        const float* x, int64_t batch, float* y, void* ws, size_t ws_bytes,
                        void* stream) {
  return kq_deploy_matvec(packed, m, n, bits, group, scales, zeros, S_X, S_G, sign_u, sign_v, mode,
                          x, batch, y, ws, ws_bytes, S(stream));
}

int kronq_quantize_layer_noalloc(float* W, int64_t m, int64_t n, const float* U_c, int bits,
                                 int group, int block, uint8_t* codes, float* scales,
                                 uint8_t* zeros, float* W_hat, int32_t* info, void* stream) {
  return kq_quantize_layer_noalloc(W, m, n, U_c, bits, group, block, codes, scales, zeros, W_hat,
                                   info, S(stream));
}

int kronq_pack(const uint8_t* codes, int64_t m, int64_t n, int bits, uint32_t* packed,
               void* stream) {
  return kq_pack(codes, m, n, bits, packed, S(stream));
}

int kronq_unpack(const uint32_t* packed, int64_t m, int64_t n, int bits, uint8_t* codes,
                 void* stream) {
  return kq_unpack(packed, m, n, bits, codes, S(stream));
}

int kronq_layer_loss(const float* W_ref, const float* W_hat, int64_t m, int64_t n,
                     const float* H_X, const float* H_G, double* loss_out, void* ws,
                     size_t ws_bytes, void* stream) {
  return kq_layer_loss(W_ref, W_hat, m, n, H_X, H_G, loss_out, ws, ws_bytes, S(stream));
}

size_t kronq_gptaq_workspace_size(int64_t m, int64_t n) {
  if (m <= 0 || n <= 0) return 0;
  size_t s = kronq_workspace_size(m, n, 4, -1, 128);
  const size_t parts[3] = {kq_drift_ws(n), kq_correction_ws(n), kq_quantize_asym_ws(m, n)};
  for (size_t p : parts)
    if (p > s) s = p;
  return s;
}

int kronq_drift_covariance(const void* XqX, int64_t N, int64_t n, int64_t ld, float* H, float* A,
                           int32_t* info, void* ws, size_t ws_bytes, void* stream) {
  return kq_drift_covariance(static_cast<const uint16_t*>(XqX), N, n, ld, H, A, info, ws, ws_bytes,
                             S(stream));
}

int kronq_biip_rotate_input(float* A, int64_t n, const float* S_X, const int8_t* sign_v, int mode,
                            void* ws, size_t ws_bytes, void* stream) {
  return kq_biip_rotate_input(A, n, S_X, sign_v, mode, ws, ws_bytes, S(stream));
}

int kronq_gptaq_correction(const float* A, const float* U_c, int64_t n, float alpha, float* P,
                           int32_t* info, void* ws, size_t ws_bytes, void* stream) {
  return kq_gptaq_correction(A, U_c, n, alpha, P, info, ws, ws_bytes, S(stream));
}

int kronq_quantize_layer_gptaq(float* W, int64_t m, int64_t n, const float* U_c, const float* P,
                               int bits, int group, int block, uint8_t* codes, float* scales,
                               uint8_t* zeros, float* W_hat, int32_t* info, void* ws,
                               size_t ws_bytes, void* stream) {
  return kq_quantize_layer_asym(W, m, n, U_c, P, bits, group, block, codes, scales, zeros, W_hat,
                                info, ws, ws_bytes, S(stream));
}

}  // extern "C"
