// Tensor-core (tcgen05) weight GEMM: placeholder until the sm_100a kernel lands.
#pragma once
#include <vector>
#include "fm_common.cuh"

namespace fm {

struct TcMap {
  bool valid = false;
};
struct TcMaps {
  TcMap embed, lm, fc;
  std::vector<TcMap> qkv, kv, o, up, down;
  TcMaps() : qkv(64), kv(64), o(64), up(64), down(64) {}
};

inline bool tc_supported(int, int, int, int) { return false; }
inline bool tc_make_maps(TcMaps&, const void*, const void*, const void*, const void* const*,
                         const void* const*, const void* const*, const void* const*, int, int, int,
                         int, int, char*, size_t) {
  return true;
}
inline void tc_free_maps(TcMaps&) {}
template <class Epi>
fm_status tc_gemm(const TcMaps&, const TcMap&, const bf16*, int, int, int, int, Epi, float*, size_t,
                  unsigned*, int, int, cudaStream_t, char*, size_t, int*) {
  return FM_ERR_UNSUPPORTED;
}
inline fm_status tc_lm_head_argmax(const TcMaps&, const bf16*, int, int, int, float*, int*, int,
                                   int, cudaStream_t, char*, size_t, int*) {
  return FM_ERR_UNSUPPORTED;
}

}  // namespace fm
