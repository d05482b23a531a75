// sink_plan.cu -- host-side slot planning for the NVFP4 KV cache under the
// two-level attention sinks of multi-shot generation.
//
// Each chunk of new frames attends to (neurohive.io LongLive-2.0 article,
// inference section on attention sinks; tailorednewshub.com LongLive-2.0
// article, section "Sumidero de Atención Multi-Toma"; 171host.com teardown,
// section 2.2):
//   G: the first global_sinks frames of the video, kept for good;
//   H: the first shot_sinks frames of the current shot, re-bound at each cut;
//   L: the last `window` frames up to and including the chunk's own.
// The planner keeps a frame -> slot map over the cache's slot pool.  For the
// next chunk it frees every slot whose frame is outside G u H u L of that
// chunk (such a frame is never attended again: G stays, H changes only at a
// cut, and L only slides forward), gives the chunk's frames the lowest free
// slots (the dst_slots of nvfp4_kv_quant_chunk), and lists the slots of
// G u H u L in frame order (the slot list of nvfp4_kv_dequant_window and
// nvfp4_window_attention).  No device work: plain host bookkeeping.
#include <algorithm>
#include <new>
#include <vector>

#include "../../include/nvfp4.h"

struct nvfp4_sink_plan {
  int32_t n_slots, global_sinks, shot_sinks, window;
  int64_t next_frame = 0;   // index of the next frame to be generated
  int64_t shot_start = 0;   // first frame of the current shot
  std::vector<int64_t> frame_of_slot;  // -1: free
};

nvfp4_sink_plan* nvfp4_sink_plan_create(int32_t n_slots, int32_t global_sinks, int32_t shot_sinks,
                                        int32_t window) {
  if (global_sinks < 0 || shot_sinks < 0 || window < 1 ||
      n_slots < int64_t(global_sinks) + shot_sinks + window ||
      n_slots > NVFP4_KV_MAX_WINDOW_SLOTS)
    return nullptr;
  nvfp4_sink_plan* p = new (std::nothrow) nvfp4_sink_plan;
  if (!p) return nullptr;
  p->n_slots = n_slots;
  p->global_sinks = global_sinks;
  p->shot_sinks = shot_sinks;
  p->window = window;
  p->frame_of_slot.assign(size_t(n_slots), -1);
  return p;
}

void nvfp4_sink_plan_destroy(nvfp4_sink_plan* plan) { delete plan; }

nvfp4_status nvfp4_sink_plan_next(nvfp4_sink_plan* p, int32_t n_frames, int32_t new_shot,
                                  int32_t* dst_slots, int32_t* window_slots, int32_t* n_window) {
  if (!p || !dst_slots || !window_slots || !n_window || n_frames < 1 ||
      n_frames > NVFP4_KV_MAX_CHUNK_FRAMES || n_frames > p->window)
    return NVFP4_ERR_INVALID_ARG;
  const int64_t f0 = p->next_frame, f1 = f0 + n_frames;  // the chunk: frames [f0, f1)
  const int64_t shot = (new_shot || f0 == 0) ? f0 : p->shot_start;
  auto attended = [&](int64_t f) {
    return f < f1 && (f < p->global_sinks || (f >= shot && f < shot + p->shot_sinks) ||
                      f >= f1 - p->window);
  };
  // free the slots of frames this chunk does not attend; then the chunk's frames
  std::vector<int64_t> slots = p->frame_of_slot;
  for (int64_t& f : slots)
    if (f >= 0 && !attended(f)) f = -1;
  int32_t k = 0;
  for (int32_t s = 0; s < p->n_slots && k < n_frames; ++s)
    if (slots[size_t(s)] < 0) {
      slots[size_t(s)] = f0 + k;
      dst_slots[k++] = s;
    }
  if (k < n_frames) return NVFP4_ERR_UNSUPPORTED_SHAPE;  // cannot happen with the create bounds
  // the attended frames' slots, in frame order
  std::vector<std::pair<int64_t, int32_t>> held;
  for (int32_t s = 0; s < p->n_slots; ++s)
    if (slots[size_t(s)] >= 0) held.emplace_back(slots[size_t(s)], s);
  std::sort(held.begin(), held.end());
  int32_t n = 0;
  for (const auto& fs : held) window_slots[n++] = fs.second;
  *n_window = n;
  p->frame_of_slot.swap(slots);
  p->shot_start = shot;
  p->next_frame = f1;
  return NVFP4_OK;
}

int64_t nvfp4_sink_plan_frame_of_slot(const nvfp4_sink_plan* p, int32_t slot) {
  if (!p || slot < 0 || slot >= p->n_slots) return -1;
  return p->frame_of_slot[size_t(slot)];
}
