"""Sliding-window cache model for the oracle (TEST INFRASTRUCTURE ONLY).

Reflex abstract: the attention context is split into static, sliding and dynamic
regions, and the sliding region takes an O(1) update per control tick. Reading (the
abstract gives no layout): the sliding region is a ring of ``n_slots`` slots and a head
index; a tick writes the new token into slot ``head`` (evicting the oldest token, which
lived there) and advances head by one modulo ``n_slots``. Logical order, oldest to
newest, is slots head, head+1, ..., head-1.
"""
from __future__ import annotations

import numpy as np


class RingModel:
    def __init__(self, slots: np.ndarray):
        """slots: [..., n_slots, D] initial contents, logical order = physical order."""
        self.slots = np.array(slots, copy=True)
        self.n = self.slots.shape[-2]
        self.head = 0

    def append(self, token: np.ndarray):
        """token: [..., D], written to the slot of the oldest entry."""
        self.slots[..., self.head, :] = token
        self.head = (self.head + 1) % self.n

    def logical(self) -> np.ndarray:
        order = [(self.head + i) % self.n for i in range(self.n)]
        return self.slots[..., order, :]
