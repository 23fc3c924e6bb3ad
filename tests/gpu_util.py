"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np


def to_device(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def unpack_words(q, d_in):
    """int32 tensor of packed words -> uint8 codes [rows, d_in]."""
    return unpack_words_np(q.cpu().numpy().view(np.uint32), d_in)


def unpack_words_np(words, d_in):
    """uint32 array of packed words [rows, d_in/8] -> codes [rows, d_in]
    (nibble j of word w is channel 8w + j)."""
    rows = words.shape[0]
    return np.stack([(words >> np.uint32(4 * j)) & np.uint32(0xF) for j in range(8)],
                    axis=-1).reshape(rows, d_in).astype(np.uint8)


def bf16_to_f64(t):
    import torch
    return t.float().cpu().numpy().astype(np.float64) if t.dtype == torch.bfloat16 else t.cpu().numpy()
