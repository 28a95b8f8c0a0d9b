// Decode-on-use pipeline over a fixed pool of decoded-weight slots.
//
// The ECF8 walkthrough (§3.2.2, "即用即解压") keeps weights compressed in
// device memory, pre-allocates a pool sized for the largest layer, lets the
// layer's forward pass trigger its decode, and reuses the pool cyclically
// with no dynamic allocation; the DFloat11 article's compute/decode pipeline
// (§4) decodes the next layers in the background while the current layer
// computes.  This object schedules exactly that with CUDA events: layer m is
// decoded into slot m % n_slots on the decode stream, after the compute
// stream has released that slot's previous layer, and the compute stream
// waits for the decode before it reads the layer.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "ecf8.h"

namespace {

struct SlotState {
  int layer = -1;              // layer decoded (or being decoded) into the slot, -1 none
  bool in_use = false;         // acquired by the compute stream and not yet released
  bool ever_released = false;  // released_ev has been recorded at least once
  cudaEvent_t decoded_ev = nullptr, released_ev = nullptr;
};

struct LayerDesc {
  std::vector<ecf8_info> infos;
  std::vector<const void*> blobs;
  std::vector<size_t> blob_sizes;
  std::vector<size_t> offsets;
};

}  // namespace

struct ecf8_pipeline {
  std::vector<LayerDesc> layers;
  std::vector<void*> slots;
  std::vector<SlotState> state;
  size_t slot_bytes = 0;
  int depth = 0;
  uint32_t max_ctas = 0;
  void* workspace = nullptr;
  size_t workspace_bytes = 0;
  int32_t* status = nullptr;
  cudaStream_t decode = nullptr;
  std::mutex lock;
  std::vector<ecf8_tensor> scratch;
};

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

// Enqueues the decode of layer m into its slot, after the compute stream's
// last release of the slot.  The slot must not be in use.
int enqueue(ecf8_pipeline* p, int m) {
  const int s = m % (int)p->slots.size();
  SlotState& st = p->state[s];
  if (st.in_use) return ECF8_ERR_ARG;  // slot still in use
  if (st.ever_released && cudaStreamWaitEvent(p->decode, st.released_ev, 0) != cudaSuccess) return ECF8_ERR_CUDA;
  const LayerDesc& L = p->layers[(size_t)m];
  p->scratch.resize(L.infos.size());
  uint8_t* base = static_cast<uint8_t*>(p->slots[(size_t)s]);
  for (size_t i = 0; i < L.infos.size(); ++i)
    p->scratch[i] = ecf8_tensor{&L.infos[i], L.blobs[i], L.blob_sizes[i], base + L.offsets[i]};
  int rc = ecf8_decode_batched_ctas(p->scratch.data(), (int)p->scratch.size(), p->workspace, p->workspace_bytes,
                                    p->status, p->decode, p->max_ctas);
  if (rc) return rc;
  if (cudaEventRecord(st.decoded_ev, p->decode) != cudaSuccess) return ECF8_ERR_CUDA;
  st.layer = m;
  return ECF8_OK;
}

}  // namespace

extern "C" {

int ecf8_pipeline_create(const ecf8_layer* layers, int n_layers, void* const* d_slots, int n_slots, size_t slot_bytes,
                         int depth, uint32_t max_ctas, void* d_workspace, size_t workspace_bytes, int32_t* d_status,
                         cudaStream_t decode_stream, ecf8_pipeline** out) {
  if (!out) return ECF8_ERR_ARG;
  *out = nullptr;
  if (!layers || n_layers < 1 || !d_slots || n_slots < 1 || depth < 0 || n_slots < depth + 1) return ECF8_ERR_ARG;
  int max_count = 0;
  for (int l = 0; l < n_layers; ++l) {
    const ecf8_layer& L = layers[l];
    if (L.count < 0 || (L.count > 0 && !L.tensors)) return ECF8_ERR_ARG;
    max_count = L.count > max_count ? L.count : max_count;
    for (int i = 0; i < L.count; ++i) {
      const ecf8_layer_tensor& t = L.tensors[i];
      if (!t.info) return ECF8_ERR_ARG;
      if (t.info->n && t.blob_size < t.info->blob_bytes) return ECF8_ERR_ARG;
      if ((t.out_offset & 15) != 0) return ECF8_ERR_ALIGN;
      if (t.out_offset > slot_bytes || t.info->n > slot_bytes - t.out_offset) return ECF8_ERR_ARG;
    }
  }
  for (int s = 0; s < n_slots; ++s)
    if (!d_slots[s] || !aligned16(d_slots[s])) return d_slots[s] ? ECF8_ERR_ALIGN : ECF8_ERR_ARG;
  const size_t ws_need = ecf8_batched_workspace_size(max_count);
  if (ws_need && (!d_workspace || workspace_bytes < ws_need)) return ECF8_ERR_WORKSPACE;
  if (d_workspace && !aligned16(d_workspace)) return ECF8_ERR_ALIGN;

  ecf8_pipeline* p = new ecf8_pipeline();
  p->layers.resize((size_t)n_layers);
  for (int l = 0; l < n_layers; ++l) {
    LayerDesc& D = p->layers[(size_t)l];
    for (int i = 0; i < layers[l].count; ++i) {
      const ecf8_layer_tensor& t = layers[l].tensors[i];
      D.infos.push_back(*t.info);
      D.blobs.push_back(t.d_blob);
      D.blob_sizes.push_back(t.blob_size);
      D.offsets.push_back(t.out_offset);
    }
  }
  p->slots.assign(d_slots, d_slots + n_slots);
  p->state.resize((size_t)n_slots);
  p->slot_bytes = slot_bytes;
  p->depth = depth;
  p->max_ctas = max_ctas;
  p->workspace = d_workspace;
  p->workspace_bytes = workspace_bytes;
  p->status = d_status;
  p->decode = decode_stream;
  for (SlotState& st : p->state) {
    if (cudaEventCreateWithFlags(&st.decoded_ev, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&st.released_ev, cudaEventDisableTiming) != cudaSuccess) {
      ecf8_pipeline_destroy(p);
      return ECF8_ERR_CUDA;
    }
  }
  *out = p;
  return ECF8_OK;
}

int ecf8_pipeline_acquire(ecf8_pipeline* p, int layer, cudaStream_t compute, void** d_weights) {
  if (!p || !d_weights || layer < 0 || layer >= (int)p->layers.size()) return ECF8_ERR_ARG;
  std::lock_guard<std::mutex> guard(p->lock);
  const int n = (int)p->slots.size();
  const int s = layer % n;
  if (p->state[(size_t)s].layer != layer) {
    int rc = enqueue(p, layer);
    if (rc) return rc;
  }
  // decode ahead: layers layer+1 .. layer+depth, each once its slot is free
  for (int m = layer + 1; m <= layer + p->depth && m < (int)p->layers.size(); ++m) {
    SlotState& st = p->state[(size_t)(m % n)];
    if (st.layer == m) continue;
    if (st.in_use) break;  // its slot is still in use: decode it at a later acquire
    int rc = enqueue(p, m);
    if (rc) return rc;
  }
  if (cudaStreamWaitEvent(compute, p->state[(size_t)s].decoded_ev, 0) != cudaSuccess) return ECF8_ERR_CUDA;
  p->state[(size_t)s].in_use = true;  // until ecf8_pipeline_release
  *d_weights = p->slots[(size_t)s];
  return ECF8_OK;
}

int ecf8_pipeline_release(ecf8_pipeline* p, int layer, cudaStream_t compute) {
  if (!p || layer < 0 || layer >= (int)p->layers.size()) return ECF8_ERR_ARG;
  std::lock_guard<std::mutex> guard(p->lock);
  SlotState& st = p->state[(size_t)(layer % (int)p->slots.size())];
  if (st.layer != layer || !st.in_use) return ECF8_ERR_ARG;
  if (cudaEventRecord(st.released_ev, compute) != cudaSuccess) return ECF8_ERR_CUDA;
  st.in_use = false;
  st.ever_released = true;
  return ECF8_OK;
}

void ecf8_pipeline_destroy(ecf8_pipeline* p) {
  if (!p) return;
  for (SlotState& st : p->state) {
    if (st.decoded_ev) cudaEventDestroy(st.decoded_ev);
    if (st.released_ev) cudaEventDestroy(st.released_ev);
  }
  delete p;
}

}  // extern "C"
