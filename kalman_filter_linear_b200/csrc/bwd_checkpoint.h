// Interval of the state checkpoints the backward pass keeps: the forward saves
// the state before every kBwdCheckpoint-th token, and the backward rebuilds
// the states in between from them (shared by the saving forward, the
// backward kernel and the workspace layout).
#pragma once

namespace kdn {
constexpr int kBwdCheckpoint = 16;
}  // namespace kdn
