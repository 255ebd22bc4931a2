// The host side of the device error flags and wait limits of ptx.cuh: each
// translation unit registers how to find its copies, and the functions here
// read and clear every flag at once (one small gather kernel, one copy, one
// synchronization) and set every limit.
#include <map>
#include <mutex>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace gwb {
namespace {

constexpr int kMaxUnits = 16;

std::vector<DeviceStateAddrs> &registry() {
  static std::vector<DeviceStateAddrs> r;   // filled while the library loads
  return r;
}

struct UnitAddrs {
  int n = 0;
  unsigned int *flag[kMaxUnits] = {};
  unsigned long long *wait[kMaxUnits] = {};
};

std::mutex g_mu;
std::map<int, UnitAddrs> g_addrs;   // per device

struct FlagList {
  unsigned int *flag[kMaxUnits];
  int n;
};

__device__ unsigned int g_gathered = 0;

// ORs every unit's flag into g_gathered and clears the flags.
__global__ void k_gather_flags(const FlagList l) {
  unsigned int v = 0;
  for (int i = 0; i < l.n; i++) v |= atomicExch(l.flag[i], 0u);
  g_gathered = v;
}

gwb_status unit_addrs(UnitAddrs *out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_addrs.find(dev);
  if (it == g_addrs.end()) {
    UnitAddrs a;
    for (DeviceStateAddrs f : registry()) {
      if (a.n == kMaxUnits) return fail(GWB_ERR_CUDA, "more than %d translation units hold device state", kMaxUnits);
      e = f(&a.flag[a.n], &a.wait[a.n]);
      if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      a.n++;
    }
    it = g_addrs.emplace(dev, a).first;
  }
  *out = it->second;
  return GWB_OK;
}

}  // namespace

void register_device_state(DeviceStateAddrs addrs) { registry().push_back(addrs); }

gwb_status read_and_clear_device_error(cudaStream_t st, unsigned int *flag) {
  UnitAddrs a;
  gwb_status s = unit_addrs(&a);
  if (s != GWB_OK) return s;
  FlagList l{};
  for (int i = 0; i < a.n; i++) l.flag[i] = a.flag[i];
  l.n = a.n;
  k_gather_flags<<<1, 1, 0, st>>>(l);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbolAsync(flag, g_gathered, sizeof(unsigned int), 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "device error check: %s", cudaGetErrorString(e));
  return GWB_OK;
}

gwb_status set_wait_cycles(unsigned long long cycles) {
  UnitAddrs a;
  gwb_status s = unit_addrs(&a);
  if (s != GWB_OK) return s;
  const unsigned long long v = cycles == 0 ? kWaitCycles : cycles;
  for (int i = 0; i < a.n; i++) {
    const cudaError_t e = cudaMemcpy(a.wait[i], &v, sizeof(v), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "setting the wait limit: %s", cudaGetErrorString(e));
  }
  return GWB_OK;
}

}  // namespace gwb
