// Internal declarations of libveda (not part of the C ABI).
#pragma once

#include <cstdint>
#include <mutex>
#include <string>
#include <vector>

#include "veda.h"

namespace veda {

constexpr int kTile = VEDA_TILE;
constexpr int kMaxDevices = 64;

// Device copy of a layout's index data, made once per device on first use.
struct DeviceCopy {
    bool ready = false;
    int32_t* perm = nullptr;         // [n_slots] packed row per slot, -1 on padding
    int32_t* valid_count = nullptr;  // [n_tiles]
    int32_t* ok_list = nullptr;      // [n_kv_ok] ascending ids of non-empty tiles
    int32_t* allowed = nullptr;      // [n_blocks * n_video]
};

// Records `msg` as the calling thread's last error and returns `code`.
int fail(int code, const std::string& msg);
void clear_error();

}  // namespace veda

struct veda_layout {
    veda_layout_desc desc{};
    std::vector<int32_t> perm;         // [n_slots]
    std::vector<int32_t> valid_count;  // [n_tiles]
    std::vector<int32_t> ok_list;      // [n_kv_ok]
    std::vector<int32_t> allowed;      // [n_blocks * n_video]
    mutable std::mutex mu;
    mutable veda::DeviceCopy dev[veda::kMaxDevices];
};
