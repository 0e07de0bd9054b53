// devcache.h -- host-side memo of per-device, per-kernel setup results.
//
// Several launch paths do a one-time setup that depends on the device the
// calling thread has current: raising a kernel's dynamic shared-memory limit
// (cudaFuncSetAttribute is per device), or asking how many CTAs of a kernel
// fit on an SM.  PerDeviceMemo keeps one result per (key, device) pair:
// computed on the first call for that pair, returned from the table after
// that, recomputed when the computation failed (a failure is never cached).
// It is thread-safe (one mutex; the computation runs under it, so each pair
// is computed once even under concurrent first calls) and holds no CUDA
// types, so the host logic is tested on a machine without a GPU.
#pragma once
#include <mutex>

namespace bsq {

template <int kCapacity>
class PerDeviceMemo {
  public:
    // compute() returns the value; ok(value) says whether to keep it.  When
    // the table is full, values are still computed and returned, uncached.
    template <class Compute, class Ok>
    int get(const void *key, int dev, Compute compute, Ok ok) {
        std::lock_guard<std::mutex> lk(mu_);
        for (int i = 0; i < n_; i++)
            if (e_[i].key == key && e_[i].dev == dev) return e_[i].value;
        const int v = compute();
        if (ok(v) && n_ < kCapacity) e_[n_++] = {key, dev, v};
        return v;
    }
    int size() {
        std::lock_guard<std::mutex> lk(mu_);
        return n_;
    }

  private:
    struct Entry {
        const void *key;
        int dev;
        int value;
    };
    std::mutex mu_;
    Entry e_[kCapacity] = {};
    int n_ = 0;
};

}  // namespace bsq
