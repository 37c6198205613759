"""A caller-owned paged latent cache and typed views of its pages.

Layouts (include/mla.h): an f32/bf16 page is [page_size][d_c + d_rope] rows
[c | k^R]; an FP8 page is [page_size][d_c] e4m3 codes, then [page_size][d_rope]
bf16 k^R, then [page_size][d_c/128] fp32 scales, each sub-block starting on a
128-byte boundary.  Token `pos` of sequence b sits in row pos % page_size of
page page_table[b, pos // page_size].  This module only places and reads rows;
it does no arithmetic on them.
"""
from __future__ import annotations

import torch

from . import binding as B


def _a128(x: int) -> int:
    return (x + 127) // 128 * 128


class PagedLatentCache:
    def __init__(self, dims: B.MlaDims, num_pages: int, device="cuda", fill: int | None = 0):
        self.dims = dims
        self.num_pages = num_pages
        self.P = dims.page_size
        self.d_c, self.d_r = dims.d_c, dims.d_rope
        self.page_bytes = self.layout_page_bytes(dims)
        lib_bytes = B.cache_page_bytes(dims)
        if lib_bytes != self.page_bytes:
            raise RuntimeError(f"page layout mismatch: {self.page_bytes} != libmla {lib_bytes}")
        n = num_pages * self.page_bytes
        self.pool = (torch.zeros(n, dtype=torch.uint8, device=device) if fill == 0 else
                     torch.empty(n, dtype=torch.uint8, device=device))
        if fill not in (0, None):
            self.pool.fill_(fill)

    @staticmethod
    def layout_page_bytes(dims) -> int:
        P, dc, dr = dims.page_size, dims.d_c, dims.d_rope
        if dims.cache_dtype == B.MLA_F32:
            return P * (dc + dr) * 4
        if dims.cache_dtype == B.MLA_BF16:
            return P * (dc + dr) * 2
        kr_off = _a128(P * dc)
        sc_off = _a128(kr_off + P * dr * 2)
        return _a128(sc_off + P * (dc // 128) * 4)

    # typed [num_pages, page_size, width] views into the byte pool
    def _view(self, dtype, byte_off, width):
        es = torch.tensor([], dtype=dtype).element_size()
        base = self.pool.view(dtype)
        return torch.as_strided(base, (self.num_pages, self.P, width), (self.page_bytes // es, width, 1),
                                byte_off // es)

    def views(self) -> dict:
        if self.dims.cache_dtype == B.MLA_FP8_E4M3:
            kr_off = _a128(self.P * self.d_c)
            sc_off = _a128(kr_off + self.P * self.d_r * 2)
            return {"codes": self._view(torch.uint8, 0, self.d_c),
                    "kr": self._view(torch.bfloat16, kr_off, self.d_r),
                    "scales": self._view(torch.float32, sc_off, self.d_c // 128)}
        dt = torch.float32 if self.dims.cache_dtype == B.MLA_F32 else torch.bfloat16
        rows = self._view(dt, 0, self.d_c + self.d_r)
        return {"c": rows[..., :self.d_c], "kr": rows[..., self.d_c:]}

    def slots(self, page_table_row: torch.Tensor, positions: torch.Tensor):
        """(page, row) index tensors for positions of one sequence."""
        pages = page_table_row.to(positions.device).long()[positions // self.P]
        return pages, positions % self.P

    def write_rows(self, page_table_row, positions, rows: dict):
        pages, r = self.slots(page_table_row, positions)
        v = self.views()
        for k, x in rows.items():
            v[k][pages, r] = x.to(v[k].dtype)

    def read_rows(self, page_table_row, positions) -> dict:
        pages, r = self.slots(page_table_row, positions)
        return {k: x[pages, r] for k, x in self.views().items()}
