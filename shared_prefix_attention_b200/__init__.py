"""Shared-prefix attention over a flat, deduplicated packed layout, for B200."""
