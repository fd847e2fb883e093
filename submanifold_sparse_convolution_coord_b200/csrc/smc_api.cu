// C ABI of libsmc (declared in include/smc.h): argument checks, the index
// handle and dispatch to the kernels.  No call here touches the CPU copy of
// any tensor, and no compute path exists outside the CUDA kernels.
#include <cstdint>
#include <new>

#include "smc_internal.h"

struct smc_index {
  int device = 0;
  int32_t stride = 1;
  int32_t order = SMC_ORDER_MASK;  // row order of the current tile plan
  smc::Plan plan;
  // workspace of the backward passes (transposed weights, partial sums),
  // grown stream-ordered; calls on one handle are stream-ordered
  void* work = nullptr;
  size_t work_bytes = 0;
  // launch configurations chosen by smc_autotune, per layer shape
  struct Tuned {
    int K, cin, cout, dtype, cfg;
  };
  static constexpr int kMaxTuned = 16;
  Tuned tuned[kMaxTuned];
  int n_tuned = 0;
  int tuned_config(int K, int cin, int cout, int dtype) const {
    for (int i = 0; i < n_tuned; ++i)
      if (tuned[i].K == K && tuned[i].cin == cin && tuned[i].cout == cout &&
          tuned[i].dtype == dtype)
        return tuned[i].cfg;
    return -1;
  }
  void set_tuned(int K, int cin, int cout, int dtype, int cfg) {
    for (int i = 0; i < n_tuned; ++i)
      if (tuned[i].K == K && tuned[i].cin == cin && tuned[i].cout == cout &&
          tuned[i].dtype == dtype) {
        tuned[i].cfg = cfg;
        return;
      }
    if (n_tuned < kMaxTuned) tuned[n_tuned++] = Tuned{K, cin, cout, dtype, cfg};
  }
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(int dtype) {
  switch (dtype) {
    case SMC_F32:
      return 4;
    case SMC_F16:
    case SMC_BF16:
      return 2;
    default:
      return 0;
  }
}

// Make the handle's workspace at least `bytes` long, stream-ordered on s.
int ensure_workspace(smc_index* h, size_t bytes, cudaStream_t s) {
  if (bytes <= h->work_bytes) return SMC_OK;
  if (h->work) smc::dev_free(h->work, s);
  h->work = nullptr;
  h->work_bytes = 0;
  bytes = (bytes + 255) & ~size_t(255);
  if (smc::dev_alloc(&h->work, bytes, s) != cudaSuccess) {
    cudaGetLastError();
    h->work = nullptr;
    return SMC_ERR_OOM;
  }
  h->work_bytes = bytes;
  return SMC_OK;
}

// Checks shared by the forward and backward calls.
int check_call(smc_index* h, int K, int cin, int cout, int dtype) {
  if (!h) return SMC_ERR_INVALID;
  // the handle's plan lives on the device it was built on; launching from
  // another current device would hand that device foreign pointers
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return SMC_ERR_CUDA;
  if (cur != h->device) return SMC_ERR_INVALID;
  if (K != 1 && K != 3) return SMC_ERR_INVALID;
  if (elem_bytes(dtype) == 0 || cin < 1 || cout < 1) return SMC_ERR_INVALID;
  return SMC_OK;
}

int conv(const smc::Plan& plan, bool dense, const void* x, const void* W, void* y, int cin,
         int cout, int dtype, const smc::Epilogue& ep, cudaStream_t s, int cfg = -1) {
  if (smc::conv_tc_supported(cin, cout, dtype))
    return smc::launch_conv_tc(plan, dense, x, W, y, cin, cout, dtype, ep, s, cfg);
  return smc::launch_conv_simt(plan, dense, x, W, y, cin, cout, dtype, ep, s);
}

}  // namespace

extern "C" {

int smc_version(void) { return 100; }

const char* smc_status_string(int status) {
  switch (status) {
    case SMC_OK:
      return "ok";
    case SMC_ERR_INVALID:
      return "invalid argument";
    case SMC_ERR_DUPLICATE:
      return "duplicate coordinate";
    case SMC_ERR_RANGE:
      return "coordinate out of range (b in [0,32768), x,y,z in [0,65536))";
    case SMC_ERR_OOM:
      return "device allocation failed";
    case SMC_ERR_CUDA:
      return "CUDA error";
    case SMC_ERR_UNSUPPORTED:
      return "unsupported shape or dtype";
    case SMC_ERR_TABLE_FULL:
      return "coordinate hash table full";
    case SMC_ERR_TIMEOUT:
      return "a device-side wait timed out";
    default:
      return "unknown status";
  }
}

int smc_build_index_ex(const int32_t* coords_dev, int64_t n, int32_t stride,
                       const smc_index_options* opts, smc_stream_t stream,
                       smc_handle_t* out_handle) {
  if (!out_handle) return SMC_ERR_INVALID;
  *out_handle = nullptr;
  if (n < 0 || stride < 1 || (n > 0 && !coords_dev)) return SMC_ERR_INVALID;
  if (n > 0 && !aligned16(coords_dev)) return SMC_ERR_INVALID;
  if (n >= (int64_t(1) << 31) / smc::kTaps) return SMC_ERR_UNSUPPORTED;
  int64_t cap = 0;
  int32_t order = SMC_ORDER_MASK, lookup = SMC_LOOKUP_HASH;
  if (opts) {
    if (opts->table_capacity < 0 ||
        (opts->order != SMC_ORDER_MASK && opts->order != SMC_ORDER_INPUT &&
         opts->order != SMC_ORDER_GREEDY) ||
        (opts->lookup != SMC_LOOKUP_HASH && opts->lookup != SMC_LOOKUP_SORT))
      return SMC_ERR_INVALID;
    cap = opts->table_capacity;
    order = opts->order;
    lookup = opts->lookup;
  }
  smc_index* h = new (std::nothrow) smc_index();
  if (!h) return SMC_ERR_OOM;
  if (cudaGetDevice(&h->device) != cudaSuccess) {
    delete h;
    return SMC_ERR_CUDA;
  }
  h->stride = stride;
  h->order = order;
  const int rc = smc::build_plan(coords_dev, n, stride, cap, order, lookup,
                                 reinterpret_cast<cudaStream_t>(stream), &h->plan);
  if (rc != SMC_OK) {
    delete h;
    return rc;
  }
  *out_handle = h;
  return SMC_OK;
}

int smc_build_index(const int32_t* coords_dev, int64_t n, int32_t stride,
                    smc_handle_t* out_handle) {
  return smc_build_index_ex(coords_dev, n, stride, nullptr, nullptr, out_handle);
}

int smc_forward_ex(smc_handle_t h, const void* feats, const void* W, void* out, int K, int cin,
                   int cout, int dtype, const smc_epilogue* ep, smc_stream_t stream) {
  const int rc = check_call(h, K, cin, cout, dtype);
  if (rc != SMC_OK) return rc;
  smc::Epilogue e;
  if (ep) {
    if (ep->reserved != 0 || ep->activation < SMC_ACT_NONE || ep->activation > SMC_ACT_GELU)
      return SMC_ERR_INVALID;
    if ((ep->bias && !aligned16(ep->bias)) || (ep->residual && !aligned16(ep->residual)))
      return SMC_ERR_INVALID;
    e.bias = ep->bias;
    e.residual = ep->residual;
    e.act = ep->activation;
  }
  const smc::Plan& plan = h->plan;
  if (plan.n == 0) return SMC_OK;
  if (!feats || !W || !out) return SMC_ERR_INVALID;
  if (!aligned16(feats) || !aligned16(W) || !aligned16(out)) return SMC_ERR_INVALID;
  return conv(plan, K == 1, feats, W, out, cin, cout, dtype, e,
              reinterpret_cast<cudaStream_t>(stream), h->tuned_config(K, cin, cout, dtype));
}

int smc_forward(smc_handle_t h, const void* feats, const void* W, void* out, int K, int cin,
                int cout, int dtype, smc_stream_t stream) {
  return smc_forward_ex(h, feats, W, out, K, cin, cout, dtype, nullptr, stream);
}

const char* smc_conv_config_name(int config) { return smc::conv_config_name(config); }

int smc_replan(smc_handle_t h, int order, smc_stream_t stream) {
  if (!h) return SMC_ERR_INVALID;
  if (order != SMC_ORDER_MASK && order != SMC_ORDER_INPUT && order != SMC_ORDER_GREEDY)
    return SMC_ERR_INVALID;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return SMC_ERR_CUDA;
  if (cur != h->device) return SMC_ERR_INVALID;
  const int rc = smc::replan(&h->plan, order, reinterpret_cast<cudaStream_t>(stream));
  if (rc != SMC_OK) return rc;
  h->order = order;
  h->n_tuned = 0;  // configurations were chosen for the previous plan
  return SMC_OK;
}

namespace {

// Time every valid tensor-core configuration of the shape on the caller's
// buffers (one warm-up, best of three); *best_cfg / *best_ms get the fastest.
int search_configs(smc_handle_t h, const void* feats, const void* W, void* out, int K, int cin,
                   int cout, int dtype, cudaStream_t s, int* best_cfg, float* best_ms) {
  const smc::Plan& plan = h->plan;
  const bool dense = K == 1;
  *best_cfg = -1;
  *best_ms = 0.f;
  cudaEvent_t ev[2];
  if (cudaEventCreate(&ev[0]) != cudaSuccess) return SMC_ERR_CUDA;
  if (cudaEventCreate(&ev[1]) != cudaSuccess) {
    cudaEventDestroy(ev[0]);
    return SMC_ERR_CUDA;
  }
  int status = SMC_OK;
  const smc::Epilogue none;
  for (int cfg = 0; cfg < smc::kConvConfigs && status == SMC_OK; ++cfg) {
    if (!smc::conv_config_valid(cfg, dense, cin, cout)) continue;
    float t = 0.f;
    for (int rep = 0; rep < 4 && status == SMC_OK; ++rep) {
      if (cudaEventRecord(ev[0], s) != cudaSuccess) status = SMC_ERR_CUDA;
      if (status == SMC_OK)
        status = smc::launch_conv_tc(plan, dense, feats, W, out, cin, cout, dtype, none, s, cfg);
      if (status == SMC_OK && (cudaEventRecord(ev[1], s) != cudaSuccess ||
                               cudaEventSynchronize(ev[1]) != cudaSuccess))
        status = SMC_ERR_CUDA;
      float ms = 0.f;
      if (status == SMC_OK && cudaEventElapsedTime(&ms, ev[0], ev[1]) != cudaSuccess)
        status = SMC_ERR_CUDA;
      if (rep == 1 || (rep > 1 && ms < t)) t = ms;  // the first run warms up
    }
    if (status == SMC_OK && (*best_cfg < 0 || t < *best_ms)) {
      *best_cfg = cfg;
      *best_ms = t;
    }
  }
  cudaEventDestroy(ev[0]);
  cudaEventDestroy(ev[1]);
  if (status != SMC_OK) return status;
  // a candidate whose bounded wait gave up leaves the choice as it was
  return smc_device_status(h, reinterpret_cast<smc_stream_t>(s));
}

}  // namespace

int smc_autotune_ex(smc_handle_t h, const void* feats, const void* W, void* out, int K, int cin,
                    int cout, int dtype, int search_orders, smc_stream_t stream,
                    int* chosen_config, int* chosen_order) {
  if (chosen_config) *chosen_config = -1;
  if (chosen_order) *chosen_order = h ? h->order : -1;
  const int rc = check_call(h, K, cin, cout, dtype);
  if (rc != SMC_OK) return rc;
  const smc::Plan& plan = h->plan;
  if (plan.n == 0 || !smc::conv_tc_supported(cin, cout, dtype)) return SMC_OK;
  if (!feats || !W || !out) return SMC_ERR_INVALID;
  if (!aligned16(feats) || !aligned16(W) || !aligned16(out)) return SMC_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int best_cfg = -1, best_order = h->order;
  float best_ms = 0.f;
  if (search_orders && K == 3) {
    // the row orders worth trying (the input order is an ablation)
    const int32_t orders[2] = {SMC_ORDER_MASK, SMC_ORDER_GREEDY};
    for (int32_t order : orders) {
      if (order != h->order) {
        const int r = smc_replan(h, order, stream);
        if (r != SMC_OK) return r;
      }
      int cfg = -1;
      float ms = 0.f;
      const int r = search_configs(h, feats, W, out, K, cin, cout, dtype, s, &cfg, &ms);
      if (r != SMC_OK) return r;
      if (cfg >= 0 && (best_cfg < 0 || ms < best_ms)) {
        best_cfg = cfg;
        best_ms = ms;
        best_order = order;
      }
    }
    if (best_order != h->order) {
      const int r = smc_replan(h, best_order, stream);
      if (r != SMC_OK) return r;
    }
  } else {
    const int r = search_configs(h, feats, W, out, K, cin, cout, dtype, s, &best_cfg, &best_ms);
    if (r != SMC_OK) return r;
  }
  if (best_cfg >= 0) {
    h->set_tuned(K, cin, cout, dtype, best_cfg);
    // leave out holding the chosen configuration's result
    const smc::Epilogue none;
    const int r = smc::launch_conv_tc(plan, K == 1, feats, W, out, cin, cout, dtype, none, s,
                                      best_cfg);
    if (r != SMC_OK) return r;
  }
  if (chosen_config) *chosen_config = best_cfg;
  if (chosen_order) *chosen_order = best_order;
  return SMC_OK;
}

int smc_autotune(smc_handle_t h, const void* feats, const void* W, void* out, int K, int cin,
                 int cout, int dtype, smc_stream_t stream, int* chosen) {
  return smc_autotune_ex(h, feats, W, out, K, cin, cout, dtype, 0, stream, chosen, nullptr);
}

int smc_backward_input(smc_handle_t h, const void* grad_out, const void* W, void* grad_in, int K,
                       int cin, int cout, int dtype, smc_stream_t stream) {
  int rc = check_call(h, K, cin, cout, dtype);
  if (rc != SMC_OK) return rc;
  const smc::Plan& plan = h->plan;
  if (plan.n == 0) return SMC_OK;
  if (!grad_out || !W || !grad_in) return SMC_ERR_INVALID;
  if (!aligned16(grad_out) || !aligned16(W) || !aligned16(grad_in)) return SMC_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int taps = K * K * K;
  rc = ensure_workspace(h, size_t(taps) * cin * cout * elem_bytes(dtype), s);
  if (rc != SMC_OK) return rc;
  // grad_in = conv(grad_out, W'), W'[k] = W[taps - 1 - k]^T: [taps][cout][cin]
  rc = smc::launch_weight_transpose(W, h->work, taps, cin, cout, dtype, s);
  if (rc != SMC_OK) return rc;
  return conv(plan, K == 1, grad_out, h->work, grad_in, cout, cin, dtype, smc::Epilogue{}, s);
}

int smc_backward_weight(smc_handle_t h, const void* feats, const void* grad_out, float* dW, int K,
                        int cin, int cout, int dtype, smc_stream_t stream) {
  int rc = check_call(h, K, cin, cout, dtype);
  if (rc != SMC_OK) return rc;
  if (!dW || !aligned16(dW)) return SMC_ERR_INVALID;
  const smc::Plan& plan = h->plan;
  if (plan.n > 0 && (!feats || !grad_out || !aligned16(feats) || !aligned16(grad_out)))
    return SMC_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool dense = (K == 1);
  rc = ensure_workspace(h, smc::bwd_weight_workspace_bytes(plan, dense, cin, cout, dtype), s);
  if (rc != SMC_OK) return rc;
  return smc::launch_bwd_weight(plan, dense, feats, grad_out, dW, cin, cout, dtype, h->work,
                                smc::wait_limit_ns(), s);
}

int smc_downsample2(const int32_t* coords_dev, int64_t n, const void* feats_dev, int c, int dtype,
                    int32_t* out_coords_dev, void* out_feats_dev, int64_t* out_n,
                    smc_stream_t stream) {
  if (!out_n || n < 0 || c < 1 || elem_bytes(dtype) == 0) return SMC_ERR_INVALID;
  *out_n = 0;
  if (n == 0) return SMC_OK;
  if (!coords_dev || !feats_dev || !out_coords_dev || !out_feats_dev) return SMC_ERR_INVALID;
  if (!aligned16(coords_dev) || !aligned16(out_coords_dev)) return SMC_ERR_INVALID;
  if (n >= (int64_t(1) << 31)) return SMC_ERR_UNSUPPORTED;
  return smc::downsample2(coords_dev, n, feats_dev, c, dtype, out_coords_dev, out_feats_dev, out_n,
                          reinterpret_cast<cudaStream_t>(stream));
}

int smc_subdivide2(const int32_t* coords_dev, int64_t n, const void* feats_dev, int c, int dtype,
                   int32_t* out_coords_dev, void* out_feats_dev, smc_stream_t stream) {
  if (n < 0 || c < 1 || elem_bytes(dtype) == 0) return SMC_ERR_INVALID;
  if (n == 0) return SMC_OK;
  if (!coords_dev || !feats_dev || !out_coords_dev || !out_feats_dev) return SMC_ERR_INVALID;
  if (!aligned16(coords_dev) || !aligned16(out_coords_dev)) return SMC_ERR_INVALID;
  if (n >= (int64_t(1) << 28)) return SMC_ERR_UNSUPPORTED;
  return smc::subdivide2(coords_dev, n, feats_dev, c, dtype, out_coords_dev, out_feats_dev,
                         reinterpret_cast<cudaStream_t>(stream));
}

int smc_get_neighbor_map(smc_handle_t h, int32_t* map_dev, smc_stream_t stream) {
  if (!h) return SMC_ERR_INVALID;
  if (h->plan.n == 0) return SMC_OK;
  if (!map_dev) return SMC_ERR_INVALID;
  return cudaMemcpyAsync(map_dev, h->plan.nbr, size_t(h->plan.n) * smc::kTaps * sizeof(int32_t),
                         cudaMemcpyDeviceToDevice,
                         reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SMC_OK
             : SMC_ERR_CUDA;
}

int smc_get_plan_stats(smc_handle_t h, int64_t* useful_pairs, int64_t* issued_rows_taps) {
  if (!h) return SMC_ERR_INVALID;
  if (useful_pairs) *useful_pairs = h->plan.useful_pairs;
  if (issued_rows_taps) *issued_rows_taps = h->plan.issued_rows_taps;
  return SMC_OK;
}

int smc_get_sizes(smc_handle_t h, int64_t* n, int64_t* n_tiles) {
  if (!h) return SMC_ERR_INVALID;
  if (n) *n = h->plan.n;
  if (n_tiles) *n_tiles = h->plan.n_tiles;
  return SMC_OK;
}

int smc_get_tile_plan(smc_handle_t h, int32_t* perm_dev, uint32_t* tile_mask_dev,
                      smc_stream_t stream) {
  if (!h) return SMC_ERR_INVALID;
  const smc::Plan& p = h->plan;
  if (p.n == 0) return SMC_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (perm_dev && cudaMemcpyAsync(perm_dev, p.perm, size_t(p.n) * sizeof(int32_t),
                                  cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return SMC_ERR_CUDA;
  if (tile_mask_dev && cudaMemcpyAsync(tile_mask_dev, p.tile_mask, size_t(p.n_tiles) * sizeof(uint32_t),
                                       cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return SMC_ERR_CUDA;
  return SMC_OK;
}

int smc_device_status(smc_handle_t h, smc_stream_t stream) {
  if (!h) return SMC_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, h->plan.status, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SMC_ERR_CUDA;
  if (v != 0 && cudaMemsetAsync(h->plan.status, 0, sizeof(int32_t), s) != cudaSuccess)
    return SMC_ERR_CUDA;
  if (v & smc::kDevTimeout) return SMC_ERR_TIMEOUT;
  return v == 0 ? SMC_OK : SMC_ERR_CUDA;
}

void smc_destroy(smc_handle_t h) {
  if (!h) return;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != h->device) cudaSetDevice(h->device);
  smc::free_plan(&h->plan);  // waits for the device first
  if (h->work) {
    smc::dev_free(h->work, nullptr);
    cudaStreamSynchronize(nullptr);
  }
  if (cur != h->device) cudaSetDevice(cur);
  delete h;
}

}  // extern "C"
